// Thin inline-PTX layer for sm_100a: mbarriers with bounded waits, TMA tile
// loads, tcgen05 (TMEM alloc, MMA, commit, loads) and UMMA shared-memory /
// instruction descriptors.  Everything here is a direct wrapper of one PTX
// instruction (or a short fixed sequence) from the public PTX ISA.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace entmax {

// ----------------------------------------------------------------- status bits
// Written with atomicOr into the first word of the caller's workspace.
enum : uint32_t {
  ST_NOT_CONVERGED = 1u << 0,  // some row's sum of p is off 1 by more than 1e-3
  ST_TIMEOUT       = 1u << 1,  // a bounded mbarrier wait gave up (kernel exited early)
  ST_RANGE         = 1u << 2,  // a score left the exactly-binnable range (|s| * n_bins >= 2^21)
  ST_BOUNDS        = 1u << 3,  // bounds-checked build only: an index fell outside its buffer
};

// ------------------------------------------------------- bounds-checked build
// Compiled with -DENTMAX_BOUNDS_CHECK, every shared-memory, tensor-memory and
// global index the kernels compute is checked against its buffer before the
// access; a violation ORs ST_BOUNDS into the status word and the access is
// skipped (a load yields zeros), so the kernel never faults or traps on it.
// Every thread of a kernel records the status word with bounds_init() before
// its first check (all write the same pointer into one block-shared slot, so
// each thread sees a valid pointer without a barrier); the checks read it from
// there.  The normal build compiles every check away.
#ifdef ENTMAX_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;
__device__ __forceinline__ uint32_t** bounds_status_slot() {
  __shared__ uint32_t* slot;
  return &slot;
}
__device__ __forceinline__ void bounds_init(uint32_t* status) {
  *reinterpret_cast<uint32_t* volatile*>(bounds_status_slot()) = status;
}
__device__ __forceinline__ bool in_bounds(bool ok) {
  if (!ok) atomicOr(*bounds_status_slot(), ST_BOUNDS);
  return ok;
}
#else
constexpr bool kBoundsCheck = false;
__device__ __forceinline__ void bounds_init(uint32_t*) {}
__device__ __forceinline__ bool in_bounds(bool) { return true; }
#endif


// A TMEM access of `ncols` 32-bit columns at taddr (lane in the upper 16 bits,
// column in the lower) stays inside the 512 columns every kernel allocates and
// in the lane quadrant of the calling warp (warp id % 4).  Warp-uniform.
__device__ __forceinline__ bool tmem_window_ok(uint32_t taddr, uint32_t ncols) {
  const uint32_t col = taddr & 0xFFFFu;
  const uint32_t lane = taddr >> 16;
  return col + ncols <= 512u && lane == 32u * ((threadIdx.x >> 5) & 3u);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Every extern __shared__ array starts at the block's dynamic shared memory.
extern __shared__ __align__(16) uint8_t entmax_dyn_smem[];

// Shared-window address one past the block's dynamic shared memory (the
// operands and TMA boxes of these kernels all live there).  The window also
// holds a reserved area and the static variables below the dynamic part, so
// the bound is the dynamic base plus its size, not the total size alone.
__device__ __forceinline__ uint32_t dyn_smem_end() {
  uint32_t sz;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(sz));
  return smem_u32(entmax_dyn_smem) + sz;
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
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

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or `hint_ns` elapse, instead of returning after the hardware's
// default limit (a waiting warp then takes no issue slots from the others).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: spins on the barrier phase until it completes, the CTA-wide
// abort flag is raised by another thread, or ~2 s of wall time pass.  Returns
// false on abort/timeout (and raises the abort flag + status bit itself on
// timeout), so no wait in these kernels can spin forever.  abort_flag and
// status may be null (teardown drains wait on time alone).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kWaitSleepNs = 20000u;   // suspend-time hint per try_wait

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (abort_flag != nullptr) *abort_flag = 1;
      if (status != nullptr) atomicOr(status, ST_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA loads
// 3-D tiled load (no multicast): coordinates are element indices, innermost
// first.  Completion is signalled on `bar` through the transaction count.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  // the innermost coordinate must be 16-byte aligned (x a multiple of 8 for
  // 2-byte elements), the box of 128 rows x 128 B lands inside shared memory on
  // the 1024-byte boundary of the 128-byte swizzle
  if (kBoundsCheck && !in_bounds((x & 7) == 0 && x >= 0 && y >= 0 && z >= 0 &&
                                 (smem_u32(smem_dst) & 1023u) == 0 &&
                                 smem_u32(smem_dst) >= smem_u32(entmax_dyn_smem) &&
                                 smem_u32(smem_dst) + 128u * 128u <= dyn_smem_end() &&
                                 smem_u32(bar) + 8u <= dyn_smem_end()))
    return;
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Generic-proxy shared-memory writes become visible to the async proxy (the
// tensor core reading an SMEM operand) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
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

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16/f16 inputs, f32 accumulate).
// The accumulator columns [d, d + N) of an M = 128 MMA (N from the
// instruction descriptor) inside the allocation, and every shared-memory
// operand starting inside the block's shared memory.
__device__ __forceinline__ bool mma_operands_ok(uint32_t d_tmem, uint32_t idesc, uint64_t a_desc,
                                                bool a_in_smem, uint64_t b_desc) {
  const uint32_t n = ((idesc >> 17) & 0x3Fu) << 3;
  const uint32_t smem = dyn_smem_end();
  const uint32_t a_addr = static_cast<uint32_t>(a_desc & 0x3FFFu) << 4;
  const uint32_t b_addr = static_cast<uint32_t>(b_desc & 0x3FFFu) << 4;
  // A in TMEM: a 128 x 16 block of 16-bit values spans 8 columns from lane 0
  const bool a_ok = a_in_smem ? a_addr < smem
                              : (static_cast<uint32_t>(a_desc) & 0xFFFFu) + 8u <= 512u &&
                                    (static_cast<uint32_t>(a_desc) >> 16) == 0u;
  return (d_tmem & 0xFFFFu) + n <= 512u && (d_tmem >> 16) == 0u && a_ok && b_addr < smem;
}

__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  if (kBoundsCheck && !in_bounds(mma_operands_ok(d_tmem, idesc, a_desc, true, b_desc))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with A read from tensor memory: row m of the 128 x 16 A block in lane m,
// its 16 values in 8 consecutive 32-bit columns from a_tmem, two per column
// (lower K index in the low half).  B stays a shared-memory descriptor.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  if (kBoundsCheck && !in_bounds(mma_operands_ok(d_tmem, idesc, a_tmem, false, b_desc))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has
// completed (their SMEM operands may then be overwritten).
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// The same MMAs and commit issued by a whole converged warp: every lane runs
// the loop that computes the (warp-uniform) descriptors and addresses, and one
// elected lane issues the instruction.  Issued from a single lane inside a
// divergent branch, the descriptors are not provably uniform and each MMA pays
// for moving them to uniform registers.
__device__ __forceinline__ void mma_f16_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  if (kBoundsCheck && !in_bounds(mma_operands_ok(d_tmem, idesc, a_desc, true, b_desc))) return;
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f16_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  if (kBoundsCheck && !in_bounds(mma_operands_ok(d_tmem, idesc, a_tmem, false, b_desc))) return;
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Warp-collective TMEM load: thread t of the warp gets 32 consecutive 32-bit
// columns of TMEM lane (lane base + t).  The warp may only address the 32-lane
// quadrant (warp id % 4).  The load and its wait sit in one asm statement so
// that no use of the registers can be scheduled before the data has arrived.
#define ENTMAX_R32(r)                                                                        \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),       \
      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),           \
      "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),           \
      "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  if (kBoundsCheck && !in_bounds(tmem_window_ok(taddr, 32))) {
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = 0u;
    return;
  }
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ENTMAX_R32(r)
      : "r"(taddr)
      : "memory");
}

// Store 16 consecutive 32-bit columns of this warp's 32 lanes (thread i ->
// lane i of its quadrant).  Complete (tmem_wait_st) before the tensor core
// reads them.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  if (kBoundsCheck && !in_bounds(tmem_window_ok(taddr, 16))) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Two 32-column loads (e.g. S and dP of the same rows) under one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t (&a)[32], uint32_t tb,
                                            uint32_t (&b)[32]) {
  if (kBoundsCheck && !in_bounds(tmem_window_ok(ta, 32) && tmem_window_ok(tb, 32))) {
#pragma unroll
    for (int e = 0; e < 32; ++e) a[e] = b[e] = 0u;
    return;
  }
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ENTMAX_R32(a), ENTMAX_R32(b)
      : "r"(ta), "r"(tb)
      : "memory");
}


// The same two loads issued without waiting; tmem_wait_ld_x2 completes them.
// Between the two calls the registers hold no data yet: only
// tmem_wait_ld_x2's outputs may be read.
__device__ __forceinline__ void tmem_ld32x2_async(uint32_t ta, uint32_t (&a)[32], uint32_t tb,
                                                  uint32_t (&b)[32]) {
  if (kBoundsCheck && !in_bounds(tmem_window_ok(ta, 32) && tmem_window_ok(tb, 32))) {
#pragma unroll
    for (int e = 0; e < 32; ++e) a[e] = b[e] = 0u;
    return;
  }
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];"
      : ENTMAX_R32(a), ENTMAX_R32(b)
      : "r"(ta), "r"(tb)
      : "memory");
}
// Waits for this thread's TMEM loads.  a and b pass through the statement as
// read-write operands, so the compiler cannot move a use of them above it.
#define ENTMAX_RW32(r)                                                                       \
  "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),       \
      "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), \
      "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),           \
      "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),           \
      "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
__device__ __forceinline__ void tmem_wait_ld_x2(uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : ENTMAX_RW32(a), ENTMAX_RW32(b) : : "memory");
}

// One 32-column load issued without waiting; tmem_wait_ld_x1 completes it.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  if (kBoundsCheck && !in_bounds(tmem_window_ok(taddr, 32))) {
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = 0u;
    return;
  }
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : ENTMAX_R32(r)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld_x1(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : ENTMAX_RW32(r) : : "memory");
}

// ---------------------------------------------------------------- descriptors
// UMMA shared-memory matrix descriptor for a 128-byte-swizzled operand whose
// tile base is 1024-byte aligned.  Fields: start address >> 4 (bits 0-13),
// leading byte offset >> 4 (16-29), stride byte offset >> 4 (32-45), fixed
// version 1 (46-47), swizzle mode 2 = 128B (61-63).
//  K-major:  rows of 128 B (64 bf16 / 32 fp32 of K), 8-row groups SBO apart;
//            LBO unused.  K steps inside a row advance the start address.
//  MN-major: 128 B of MN per row, K rows 128 B apart, 8-row K groups SBO
//            apart, further 128-byte MN slabs LBO apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Instruction descriptor for kind::f16 / kind::tf32 with f32 accumulation.
//   a_fmt/b_fmt: 0 = f16, 1 = bf16, 2 = tf32.  a_mn/b_mn: 1 = MN-major operand.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t M, uint32_t N, uint32_t a_fmt,
                                                  uint32_t b_fmt, uint32_t a_mn, uint32_t b_mn) {
  return (1u << 4)              // D format f32
         | (a_fmt << 7) | (b_fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}


}  // namespace entmax
