// common.cuh - sm_100a building blocks shared by the MLRA decode kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 MMA / TMEM access, UMMA shared-memory
// descriptors, and the split planner (the rule that cuts sequences into per-group tile runs).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlra {

constexpr int kPage = 64;    // tokens per cache page
constexpr int kTile = 128;   // tokens per decode tile (two pages, the MMA M extent)

// Device status codes (same values as mlra_status).
enum : int { kOk = 0, kErrPageOob = -4, kErrTimeout = -5, kErrSeqLen = -7, kErrDrain = -9 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// First error wins.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}
// A failed teardown drain overrides any other code: after it the context may be unusable.
__device__ __forceinline__ void force_status(int* status, int code) {
  if (status != nullptr) atomicExch(status, code);
}

// Errors found while the call's status word may not yet be cleared. The first kernel of a
// call clears the status word from one CTA after the previous kernel in the stream has
// finished; its other CTAs may fail before that clear. They never write the status word:
// they store the call's tag (a number unique to each host call, never 0) into a tag word of
// the workspace, one word per error kind, and a later kernel of the same call, which runs
// after the first has completed, turns a matching tag into the status code. A tag left in
// the word by an earlier call never matches.
struct EarlyTags {
  unsigned* words;  // 4 words in the call's workspace (kinds below)
  unsigned tag;     // this call's tag
};
enum : int { kTagTimeout = 0, kTagDrain = 1, kTagSeqLen = 2, kTagPageOob = 3 };
__device__ __forceinline__ void report_early(const EarlyTags& t, int which) {
  if (t.words != nullptr) atomicExch(t.words + which, t.tag);
}
// The first kernel's clearing CTA: status word to 0, and every tag word that does not hold
// this call's tag to 0 (a compare-and-swap, so a tag another CTA has just written survives;
// afterwards no word holds stale bits that could equal a later call's tag).
__device__ __forceinline__ void clear_status_and_tags(int* status, const EarlyTags& t) {
  if (status != nullptr) *status = 0;
  if (t.words == nullptr) return;
  for (int k = 0; k < 4; ++k) {
    const unsigned w = *reinterpret_cast<volatile unsigned*>(t.words + k);
    if (w != t.tag) atomicCAS(t.words + k, w, 0u);
  }
}
// Called by one thread of a later kernel of the same call, after griddepcontrol.wait.
__device__ __forceinline__ void fold_early(const EarlyTags& t, int* status) {
  if (t.words == nullptr) return;
  const volatile unsigned* w = t.words;
  if (w[kTagDrain] == t.tag) {
    force_status(status, kErrDrain);
    return;
  }
  if (w[kTagTimeout] == t.tag) set_status(status, kErrTimeout);
  if (w[kTagSeqLen] == t.tag) set_status(status, kErrSeqLen);
  if (w[kTagPageOob] == t.tag) set_status(status, kErrPageOob);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// Timeline trace points. They compile to nothing unless MLRA_TRACE is defined (a profiling
// build); then point `id` of kernel `k` in this CTA records %globaltimer into g_mlra_trace.
// A kernel with trace points starts with MLRA_TRACE_INIT, which reads the buffer pointer once.
#ifdef MLRA_TRACE
__device__ unsigned long long* g_mlra_trace;
constexpr int kTracePoints = 512;
#define MLRA_TRACE_INIT unsigned long long* const mlra_trace_buf_ = g_mlra_trace;
#define MLRA_TRACE_POINT(k, id)                                                                 \
  do {                                                                                          \
    const unsigned long long ts_ = global_timer_ns();                                           \
    if (mlra_trace_buf_ != nullptr && (id) < kTracePoints)                                      \
      mlra_trace_buf_[((size_t)(k) * 1024 + blockIdx.x + blockIdx.y * gridDim.x) * kTracePoints + \
                      (id)] = ts_;                                                              \
  } while (0)
#else
#define MLRA_TRACE_INIT
#define MLRA_TRACE_POINT(k, id) \
  do {                          \
  } while (0)
#endif
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// ------------------------------------------------------------------------------------
// Programmatic dependent launch
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------
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
// Suspends the thread until the phase with the given parity has completed or, at most, about
// kSuspendHintNs has passed (the hint bounds the suspension; completion wakes the thread at
// once). A long hint keeps waiting warps from spinning through issue slots that the working
// warps of the SM need.
constexpr uint32_t kSuspendHintNs = 200000;
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Non-blocking test (never suspends the thread); the teardown drain polls with it.
__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity of `bar` has completed. Gives up, raising the
// CTA's abort flag, once `limit_ns` has passed or another role raised the flag. Returns false
// when it gave up. Every wait in these kernels goes through here, so no wait is endless.
// The wait is mbarrier.try_wait, which suspends the warp in hardware until the phase completes
// (or a short hardware time limit passes), so a waiter wakes as soon as its data is there and
// leaves its issue slots to the other warps meanwhile. The limit is counted in SM cycles at
// kCyclesPerNs, i.e. at least `limit_ns` of wall time at clocks up to 2 GHz.
constexpr uint64_t kCyclesPerNs = 2;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = clock64();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kCyclesPerNs * limit_ns) {
      *abort_flag = 1;
      return false;
    }
  }
}

// Teardown wait: ignores the abort flag (in-flight copies and MMAs must land before their
// shared memory or TMEM is released) but still gives up after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_poll(bar, parity)) {
    __nanosleep(32);
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ------------------------------------------------------------------------------------
// Named barriers among a subset of warps
// ------------------------------------------------------------------------------------
// Arrives at named barrier `id` without waiting (the producer side of a hand-off).
__device__ __forceinline__ void named_bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Barrier over `threads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return out != 0;
}

// ------------------------------------------------------------------------------------
// TMA (tiled bulk tensor copies, global -> shared, completion counted on an mbarrier)
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// x: innermost coordinate (elements), y: row. x * elem_size is a multiple of 16 bytes at
// every call site (column offsets are multiples of 16 elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy (tensor core reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------------------
// tcgen05: tensor memory and MMA
// ------------------------------------------------------------------------------------
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
// D(tmem) (+)= A(smem desc) * B(smem desc), bf16 inputs, fp32 accumulate. One thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc), E4M3 inputs (K = 32 per instruction), fp32
// accumulate. One thread issues.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on `bar` once every tcgen05 MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// Loads / stores N (8, 16, 32 or 64) consecutive fp32 columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_load_row(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 8 || N == 16 || N % 32 == 0, "row width");
  if constexpr (N == 8) {
    uint32_t r[8];
    tmem_ld8(taddr, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  } else if constexpr (N == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  } else {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + 32 * c, r);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[32 * c + i] = __uint_as_float(r[i]);
    }
  }
}
template <int N>
__device__ __forceinline__ void tmem_store_row(uint32_t taddr, const float (&v)[N]) {
  if constexpr (N == 8) {
    uint32_t r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = __float_as_uint(v[i]);
    tmem_st8(taddr, r);
  } else if constexpr (N == 16) {
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i]);
    tmem_st16(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[32 * c + i]);
      tmem_st32(taddr + 32 * c, r);
    }
  }
}

// TMEM address of lane `lane`, column `col` relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, int lane, int col) {
  return base + (static_cast<uint32_t>(lane) << 16) + static_cast<uint32_t>(col);
}

// ------------------------------------------------------------------------------------
// UMMA operand descriptors
// ------------------------------------------------------------------------------------
// Layout codes of the descriptor's 3-bit swizzle field, by the byte width of one swizzled
// row: 128 -> 128-byte swizzle, 64 -> 64-byte, 32 -> 32-byte.
__host__ __device__ constexpr uint32_t swizzle_code(int row_bytes) {
  return row_bytes == 128 ? 2u : (row_bytes == 64 ? 4u : 6u);
}

// Shared-memory matrix descriptor: start address, leading / stride byte offsets (16-byte
// units), fixed version bits 46..47 = 1, swizzle mode in bits 61..63.
//   K-major operand (rows of the M/N dimension, K contiguous): SBO = byte distance between
//   consecutive groups of 8 rows; LBO unused for swizzled layouts.
//   MN-major operand (M/N contiguous, one swizzled row per K index): LBO = byte distance
//   between consecutive swizzle-width chunks of M/N; SBO = distance between groups of 8 K rows.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

// Instruction descriptor for kind::f16 with bf16 A and B and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0) and an fp32
// accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of logical byte `off` inside a swizzled region whose rows are `row_bytes`
// wide (the pattern the TMA engine writes and the tensor core reads): the 16-byte chunk
// index bits [4, 4+b) are XORed with address bits [7, 7+b), b = log2(row_bytes / 16).
__device__ __forceinline__ uint32_t swizzle(uint32_t off, int row_bytes) {
  const uint32_t mask = row_bytes == 128 ? 7u : (row_bytes == 64 ? 3u : 1u);
  return off ^ (((off >> 7) & mask) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// E4M3 conversions (round to nearest even, saturating at +-448). The first argument of the
// two-element forms lands in the lower byte, i.e. first in memory.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t e4m3x2_from_f16x2(uint32_t h2) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(h2));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t e2) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(e2));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_from_f32(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t sub_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Two non-negative values as a pair of E4M3 terms each, value ~= hi + lo: hi is the nearest
// E4M3 value, lo the nearest to the remainder (about 7 significant bits in all). The split
// goes through f16 (exact for every E4M3 value; 11 bits for the input).
__device__ __forceinline__ void e4m3x2_split(float a, float b, uint16_t& hi, uint16_t& lo) {
  const uint32_t v = f16x2_from_f32(a, b);
  hi = e4m3x2_from_f16x2(v);
  lo = e4m3x2_from_f16x2(sub_f16x2(v, f16x2_from_e4m3x2(hi)));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------------------------
// Split planner
// ------------------------------------------------------------------------------------
// The decode work is the flattened list of (sequence b, 128-token tile) pairs. With
// tiles_b = ceil(n_b / 128), T = sum_b tiles_b and quota = ceil(T / groups), group g takes
// flattened tiles [g*quota, min((g+1)*quota, T)). A run that crosses sequence boundaries
// is one segment per sequence; segment (b, g) writes its partial result to slot b + g,
// which is unique because b and g never decrease along the flattened order.

struct Segment {
  int b;           // sequence
  int tile_begin;  // first tile of sequence b in this segment
  int tile_end;    // one past the last tile
  int n;           // tokens of sequence b
};

__device__ __forceinline__ int clamp_len(int n, int cap, int* err) {
  if (n < 0 || n > cap) {
    *err = kErrSeqLen;
    return n < 0 ? 0 : cap;
  }
  return n;
}
__device__ __forceinline__ int tiles_of(int n) { return (n + kTile - 1) / kTile; }

// Block-wide sum over all sequences of tiles_b. `scratch` holds >= 32 ints. All threads of
// the block call it and get the total. `err` (per thread) collects a bad-length code.
__device__ __forceinline__ int block_total_tiles(const int* __restrict__ seq_lens, int batch,
                                                 int cap, int* scratch, int* err) {
  int local = 0;
  for (int b = threadIdx.x; b < batch; b += blockDim.x)
    local += tiles_of(clamp_len(__ldg(seq_lens + b), cap, err));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  __syncthreads();
  if (lane_id() == 0) scratch[warp_id()] = local;
  __syncthreads();
  int total = 0;
  const int nw = (blockDim.x + 31) / 32;
  for (int w = 0; w < nw; ++w) total += scratch[w];
  __syncthreads();
  return total;
}

// Block-wide exclusive scan of tiles_b over the sequences [b0, b0 + blockDim.x): returns this
// thread's prefix (relative to b0) and, via *chunk_total, the chunk's sum. scratch >= 33 ints.
__device__ __forceinline__ int block_scan_tiles(int my_tiles, int* scratch, int* chunk_total) {
  int x = my_tiles;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane_id() >= o) x += y;
  }
  __syncthreads();
  if (lane_id() == 31) scratch[warp_id()] = x;
  __syncthreads();
  int warp_prefix = 0, total = 0;
  const int nw = (blockDim.x + 31) / 32;
  for (int w = 0; w < nw; ++w) {
    if (w < warp_id()) warp_prefix += scratch[w];
    total += scratch[w];
  }
  __syncthreads();
  *chunk_total = total;
  return warp_prefix + x - my_tiles;
}

// Collects (in order) the segments of the flattened range [lo, hi), starting the walk at
// sequence `b_start` whose flattened start is `p_start` (<= lo is allowed). Writes at most
// `cap_list` segments to `list` (shared memory) and returns the count. *more is set when the
// list filled up before the range ended; then (*resume_b, *resume_p) is where to continue.
// All threads of the block must call it with the same arguments. scratch >= 40 ints.
__device__ __forceinline__ int block_collect_segments(const int* __restrict__ seq_lens, int batch,
                                                      int cap_len, int lo, int hi, int b_start,
                                                      int p_start, Segment* list, int cap_list,
                                                      int* scratch, int* more, int* resume_b,
                                                      int* resume_p, int* err) {
  int count = 0;
  int running = p_start;
  int full = 0;
  int res_b = batch, res_p = running;
  for (int base = b_start; base < batch; base += blockDim.x) {
    if (running >= hi) break;
    const int b = base + threadIdx.x;
    const int n = b < batch ? clamp_len(__ldg(seq_lens + b), cap_len, err) : 0;
    const int t = tiles_of(n);
    int chunk_total;
    const int pb = running + block_scan_tiles(t, scratch, &chunk_total);
    const bool hit = t > 0 && pb < hi && pb + t > lo;
    // ordinal of this segment among the chunk's hits
    int ord_total;
    const int ord = block_scan_tiles(hit ? 1 : 0, scratch, &ord_total);
    if (hit && count + ord < cap_list) {
      Segment s;
      s.b = b;
      s.tile_begin = max(lo, pb) - pb;
      s.tile_end = min(hi, pb + t) - pb;
      s.n = n;
      list[count + ord] = s;
    }
    // first hit that did not fit: where to resume
    if (hit && count + ord == cap_list) {
      scratch[34] = b;
      scratch[35] = pb;
    }
    __syncthreads();
    if (count + ord_total > cap_list) {
      full = 1;
      res_b = scratch[34];
      res_p = scratch[35];
      count = cap_list;
      break;
    }
    count += ord_total;
    running += chunk_total;
    __syncthreads();
  }
  __syncthreads();
  *more = full;
  *resume_b = res_b;
  *resume_p = res_p;
  return count;
}

constexpr int kPlanPer = 8;  // sequences per lane in the warp-level plan

// Warp-level planning for batches up to 32 * kPlanPer sequences: every warp that needs the
// plan computes it on its own (one read of seq_lens, a 5-step shuffle scan), with no block
// barrier, so warps do not wait on one another. Lane l owns sequences [l*per, (l+1)*per).
struct WarpPlan {
  int n[kPlanPer];  // clamped lengths of the lane's sequences
  int per, base;
  int excl;         // flattened first tile of the lane's first sequence
  int total;        // T = sum of tiles over all sequences (same in every lane)
};

// All lanes call it. Returns false (and loads nothing) when the batch is too large.
__device__ __forceinline__ bool warp_plan_load(const int* __restrict__ seq_lens, int batch, int cap_len,
                                               WarpPlan& wp, int* err) {
  wp.per = (batch + 31) / 32;
  if (wp.per > kPlanPer) return false;
  wp.base = lane_id() * wp.per;
  int local = 0;
#pragma unroll
  for (int i = 0; i < kPlanPer; ++i) {
    const int b = wp.base + i;
    wp.n[i] = (i < wp.per && b < batch) ? clamp_len(__ldg(seq_lens + b), cap_len, err) : 0;
    local += tiles_of(wp.n[i]);
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane_id() >= o) incl += y;
  }
  wp.excl = incl - local;
  wp.total = __shfl_sync(0xffffffffu, incl, 31);
  return true;
}

// Flattened first tile of sequence b (warp-uniform, 0 <= b < batch) and its tile count.
__device__ __forceinline__ int warp_plan_start(const WarpPlan& wp, int b, int* tiles) {
  int before = wp.excl, t = 0;
#pragma unroll
  for (int i = 0; i < kPlanPer; ++i) {
    const int ti = tiles_of(wp.n[i]);
    if (wp.base + i < b) before += ti;
    if (wp.base + i == b) t = ti;
  }
  const int owner = b / wp.per;
  *tiles = __shfl_sync(0xffffffffu, t, owner);
  return __shfl_sync(0xffffffffu, before, owner);
}

// Segments of the flattened tile range [lo, hi) from a warp plan, in sequence order (the same
// list block_collect_segments builds). One warp calls it. Writes at most cap_list entries and
// returns how many segments the range holds; when that exceeds cap_list, (*resume_b,
// *resume_p) name the first segment left out and its flattened start, for
// block_collect_segments to continue from.
__device__ __forceinline__ int warp_plan_segments(const WarpPlan& wp, int lo, int hi, Segment* list, int cap_list,
                                                  int* resume_b, int* resume_p) {
  int hits = 0;
  int pb = wp.excl;
#pragma unroll
  for (int i = 0; i < kPlanPer; ++i) {
    const int t = tiles_of(wp.n[i]);
    if (i < wp.per && t > 0 && pb < hi && pb + t > lo) ++hits;
    pb += t;
  }
  int incl = hits;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane_id() >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int ord = incl - hits;
  int res_b = 0, res_p = 0;
  bool found = false;
  pb = wp.excl;
#pragma unroll
  for (int i = 0; i < kPlanPer; ++i) {
    const int t = tiles_of(wp.n[i]);
    if (i < wp.per && t > 0 && pb < hi && pb + t > lo) {
      if (ord < cap_list) {
        Segment sg;
        sg.b = wp.base + i;
        sg.tile_begin = max(lo, pb) - pb;
        sg.tile_end = min(hi, pb + t) - pb;
        sg.n = wp.n[i];
        list[ord] = sg;
      } else if (ord == cap_list) {
        res_b = wp.base + i;
        res_p = pb;
        found = true;
      }
      ++ord;
    }
    pb += t;
  }
  const unsigned m = __ballot_sync(0xffffffffu, found);
  if (m) {
    const int src = __ffs(m) - 1;
    *resume_b = __shfl_sync(0xffffffffu, res_b, src);
    *resume_p = __shfl_sync(0xffffffffu, res_p, src);
  }
  return total;
}

}  // namespace mlra
