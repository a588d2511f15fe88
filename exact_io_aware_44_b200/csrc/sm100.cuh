// sm100.cuh -- thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers with bounded waits, TMA tiled loads, Tensor Memory allocation,
// tcgen05.mma (bf16 in, fp32 accumulate), tcgen05.ld/st and their fences,
// and the shared-memory / instruction descriptors tcgen05.mma reads.
//
// Descriptor bit layouts follow the PTX ISA's tcgen05 "matrix descriptor" and
// "instruction descriptor" tables for .kind::f16.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

// ----------------------------------------------------------------------------
// device status word and bounded waits
// ----------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Keep the first error: later ones do not overwrite it.
__device__ __forceinline__ void record_error(int* status, int code) { atomicCAS(status, 0, code); }

// Per-CTA context of the bounded waits. `status` is the library's device
// status word; `abort_flag` (shared memory) makes every other wait of the CTA
// give up at once after the first one ran out.
struct WaitCtx {
  volatile int* abort_flag;
  int* status;
  uint64_t budget_ns;
};

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase of `bar` with parity `parity` has completed. Returns
// false (and records FA_ERR_DEVICE_TIMEOUT) if it did not within the budget,
// or if another wait of this CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  // Second bound in case the timer does not advance: every iteration takes
  // well over 8 ns, so this cap is never reached before the time budget.
  const uint64_t max_iter = w.budget_ns / 8 + 1024;
  for (uint64_t i = 0; i < max_iter; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if (*w.abort_flag) return false;
    if (globaltimer_ns() - t0 > w.budget_ns) break;
  }
  *w.abort_flag = 1;
  record_error(w.status, FA_ERR_DEVICE_TIMEOUT);
  return false;
}

// Suspension cap of the many-thread consumer waits (softmax / elementwise
// warpgroups). Without a cap a waiter may sleep far past the phase completion.
#ifndef FA_CONSUMER_POLL_NS
#define FA_CONSUMER_POLL_NS 200
#endif
constexpr uint32_t kConsumerPollNs = FA_CONSUMER_POLL_NS;

// One poll that may suspend the thread for at most `ns` nanoseconds.
__device__ __forceinline__ bool mbar_try_wait_ns(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// As mbar_wait, with each suspension capped at `ns` nanoseconds: bounds how
// long a waiter can sleep past the phase completion while polling rarely.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, const WaitCtx& w, uint32_t ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_ns(a, parity, ns)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t max_iter = w.budget_ns / 8 + 1024;
  for (uint64_t i = 0; i < max_iter; ++i) {
    if (mbar_try_wait_ns(a, parity, ns)) return true;
    if ((i & 15) == 15) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.budget_ns) break;
    }
  }
  *w.abort_flag = 1;
  record_error(w.status, FA_ERR_DEVICE_TIMEOUT);
  return false;
}

// How the many-thread consumer roles wait for a phase (all lanes of the warp call it
// together; the result is the same on every lane):
//   0  every lane polls with try_wait (suspending for at most kConsumerPollNs)
//   1  every lane spins on test_wait
//   2  lane 0 polls with try_wait, the others meet it at __syncwarp
//   3  lane 0 spins on test_wait, the others meet it at __syncwarp
//   4  every lane probes with test_wait and sleeps kConsumerPollNs between probes
// In modes 2 and 3 the warp barrier orders the other lanes after lane 0's acquire.
#ifndef FA_CONSUMER_WAIT_MODE
#define FA_CONSUMER_WAIT_MODE 0
#endif
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtx& w);
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, const WaitCtx& w, uint32_t ns);
__device__ __forceinline__ bool consumer_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
#if FA_CONSUMER_WAIT_MODE == 0
  return mbar_wait_ns(bar, parity, w, kConsumerPollNs);
#elif FA_CONSUMER_WAIT_MODE == 1
  return mbar_wait_spin(bar, parity, w);
#elif FA_CONSUMER_WAIT_MODE == 4
  return mbar_wait_sleep(bar, parity, w, kConsumerPollNs);
#else
  bool ok = false;
  if ((threadIdx.x & 31) == 0) {
#if FA_CONSUMER_WAIT_MODE == 2
    ok = mbar_wait_ns(bar, parity, w, kConsumerPollNs);
#else
    ok = mbar_wait_spin(bar, parity, w);
#endif
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok;
#endif
}

// Non-suspending probe of a phase (mbarrier.test_wait).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_wait, but the thread never suspends: for the single-warp roles (MMA
// issue, TMA production) whose wake-up latency is on the critical path. A
// suspended try_wait can sleep on the order of a microsecond past the phase
// completion, which idles the tensor core; a spinning warp costs only its own
// issue slots. Many-thread waiters keep mbar_wait.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t max_iter = w.budget_ns / 8 + 1024;  // every probe takes well over 8 ns
  for (uint64_t i = 0; i < max_iter; ++i) {
    if (mbar_test_wait(a, parity)) return true;
    if ((i & 63) == 63) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.budget_ns) break;
    }
  }
  *w.abort_flag = 1;
  record_error(w.status, FA_ERR_DEVICE_TIMEOUT);
  return false;
}

// A whole warp waits for a phase on behalf of one lane (MMA issuer, producer): with
// FA_WARP_SPIN_LANE0 only lane 0 polls and the others meet it at the shuffle;
// otherwise every lane polls. Every lane of the warp must call it; the result is
// the same on all lanes.
#ifndef FA_WARP_SPIN_LANE0
#define FA_WARP_SPIN_LANE0 0
#endif
__device__ __forceinline__ bool warp_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
#if FA_WARP_SPIN_LANE0
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_spin(bar, parity, w);
  return __shfl_sync(0xffffffffu, ok, 0);
#else
  return mbar_wait_spin(bar, parity, w);
#endif
}

// As mbar_wait_spin, with a nanosleep of about `ns` between probes, which gives the
// issue slots back to the other warps of the sub-partition while waiting.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, const WaitCtx& w, uint32_t ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t max_iter = w.budget_ns / 8 + 1024;  // every probe takes well over 8 ns
  for (uint64_t i = 0; i < max_iter; ++i) {
    __nanosleep(ns);
    if (mbar_test_wait(a, parity)) return true;
    if ((i & 15) == 15) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.budget_ns) break;
    }
  }
  *w.abort_flag = 1;
  record_error(w.status, FA_ERR_DEVICE_TIMEOUT);
  return false;
}

// ----------------------------------------------------------------------------
// proxy / tcgen05 ordering fences
// ----------------------------------------------------------------------------

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ----------------------------------------------------------------------------
// TMA
// ----------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load of one box into shared memory; completion is signalled on `bar`
// as transaction bytes. x (innermost) must be a multiple of 8 bf16 elements.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled reduction of one shared-memory box into global memory: every element
// of the box is added (fp32 add, done by the TMA unit at L2) to the tensor at
// (x, y, z). Elements outside the tensor's bounds are skipped. Tracked by the
// issuing thread's bulk async-groups; the shared source must not be rewritten
// before bulk_wait_read() says the unit has read it.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every bulk group this thread committed has completed (writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Barrier over `count` threads (a multiple of 32) on hardware barrier `id` (1..15;
// 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ----------------------------------------------------------------------------
// Tensor Memory
// ----------------------------------------------------------------------------

// Warp-wide: allocate `ncols` (power of two >= 32) TMEM columns; the base
// address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// ----------------------------------------------------------------------------
// tcgen05.mma, kind::f16 (bf16 x bf16 -> fp32), both operands in shared memory
// ----------------------------------------------------------------------------

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f8f6f4 with E4M3 A and B (fp32 accumulate); K = 32 per instruction.
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with A in Tensor Memory: 32-bit column c holds k = 4c .. 4c + 3, lowest k in the low byte.
__device__ __forceinline__ void mma_e4m3_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor, kind::f8f6f4: fp32 accumulator, E4M3 A and B (format 0).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Same, with the A operand in Tensor Memory (128 lanes = M rows; 32-bit column c
// holds the bf16 pair k = 2c (low half), 2c + 1; a K = 16 step spans 8 columns).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B.
// bits [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
// bit 15 A major (0 = K, 1 = MN), bit 16 B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor with the 128-byte swizzle.
// bits [0,14) start >> 4, [16,30) leading byte offset >> 4, [32,46) stride
// byte offset >> 4, bit 46 version (1 on sm_100), [61,64) layout (2 = SW128).
//
// K-major tile: rows of 64 bf16 (128 B) at a 128 B pitch, 8-row atoms of
// 1024 B. SBO = 1024 B between 8-row groups; LBO is not used by swizzled
// K-major layouts. The K slice [16k, 16k+16) of a 64-wide column block
// starts 32k bytes into the atom.
//
// MN-major tile: each row holds 64 consecutive MN elements (128 B), rows
// step along K. SBO = 1024 B between groups of 8 K rows; LBO = distance
// between consecutive 64-element MN blocks.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Advance a descriptor's start address by `bytes` (a multiple of 16). Shared
// addresses are below 2^18, so start >> 4 stays below 2^14 and the add never
// carries out of the 14-bit field.
// The add is an opaque asm statement so that the compiler computes it next to
// the MMA instead of hoisting every (base + constant) descriptor of an
// unrolled loop into registers.
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
  uint64_t r;
  asm volatile("add.u64 %0, %1, %2;" : "=l"(r) : "l"(desc), "l"((uint64_t)(bytes >> 4)));
  return r;
}

// ----------------------------------------------------------------------------
// tcgen05.ld / tcgen05.st, shape 32x32b: thread t of the warp owns TMEM lane
// (warp's lane quarter) + t and N consecutive 32-bit columns.
// ----------------------------------------------------------------------------

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld; the registers are tied in so
// that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
        "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
        "+r"(r[30]), "+r"(r[31])::"memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------------------------------
// register reallocation between warpgroups (all warps of a warpgroup execute
// the same one). The shares must add up to at most the launch's threads x
// registers. .dec must lower and .inc must raise the count the warp holds
// (the launch count, `kLaunch`); anything else is undefined, hence the checks.
// ----------------------------------------------------------------------------
template <int N, int kLaunch>
__device__ __forceinline__ void regs_dec() {
  static_assert(N % 8 == 0 && N >= 24 && N < kLaunch, "setmaxnreg.dec must lower the register count");
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N, int kLaunch>
__device__ __forceinline__ void regs_inc() {
  static_assert(N % 8 == 0 && N <= 256 && N > kLaunch, "setmaxnreg.inc must raise the register count");
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ----------------------------------------------------------------------------
// small math helpers
// ----------------------------------------------------------------------------

// 2^x on the SFU (MUFU.EX2), flushing denormal results to zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32x2 arithmetic (one instruction for two lanes of work). A 64-bit
// operand holds {lo, hi} as two consecutive 32-bit registers.
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
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// 2^x for two values on the FMA and integer pipes instead of the SFU. With
// n = rint(x) (adding 1.5 * 2^23 rounds to an integer in round-to-nearest) and
// f = x - n in [-1/2, 1/2], 2^x = 2^n * 2^f: 2^f comes from a cubic whose
// coefficients were fitted for minimum maximum relative error on that interval
// (iteratively reweighted least squares; measured maximum 7.6e-5 in fp32
// Horner form), and n is added to the exponent field. Inputs are clamped at -125
// so the result stays a normal number (2^-125 instead of an underflow to 0);
// x must not be +inf or NaN.
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t r2 = f2_pack(kRound, kRound);
  const uint64_t t = f2_add(x, r2);
  const uint64_t f = f2_sub(x, f2_sub(t, r2));
  uint64_t p = f2_fma(f2_pack(0.05517052486538887f, 0.05517052486538887f), f,
                      f2_pack(0.24260830879211426f, 0.24260830879211426f));
  p = f2_fma(p, f, f2_pack(0.693260908126831f, 0.693260908126831f));
  p = f2_fma(p, f, f2_pack(0.9999282360076904f, 0.9999282360076904f));
  float t0, t1, p0, p1;
  f2_unpack(t, t0, t1);
  f2_unpack(p, p0, p1);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// max of three
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Four fp32 values to E4M3 (round to nearest, saturating), packed low byte first.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Byte offset of the 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled tile whose rows are 128 bytes apart: chunk index XOR row % 8.
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace fa
