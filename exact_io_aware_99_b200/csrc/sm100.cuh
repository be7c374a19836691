// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features
// the attention kernels use: mbarriers with bounded waits, TMA tile loads,
// tcgen05 tensor-memory allocation, MMA, commit, loads and stores.
//
// Every wait is bounded: it gives up after a time limit, records a site code
// in a device status word and raises a CTA-local abort flag, so a kernel that
// loses a producer or consumer returns instead of hanging the GPU.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>

namespace fa {

struct WaitCtl {
  int* status;                 // device status word (first timeout wins)
  unsigned long long limit_ns; // time limit of one wait
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

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

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  // No suspend-time hint: with a 20 us hint the MMA issuer came back from
  // waits on barriers that had already completed a couple of hundred cycles
  // late, and the tensor pipe, which the single issuing thread keeps only a
  // few instructions ahead, idled meanwhile (measured on B200: +3-7 % for
  // the backward without the hint, the forward unchanged).
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed.
// Returns false (and raises *abort) when the CTA is aborting or the time
// limit ran out; in the latter case `site` is recorded in the status word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const WaitCtl& ctl, int site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(a, parity)) return true;
    if ((it & 31u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        atomicCAS(ctl.status, 0, site);
        *abort = 1;
        return false;
      }
    }
  }
}

// -------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load (no multicast) of box {x..x+bx, y..y+by, z} into shared
// memory; completion is signalled as transaction bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* m, uint64_t* bar, void* dst,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ------------------------------------------------- cluster launch control

// Ask the hardware to cancel the launch of a CTA of this grid that has not
// started yet (sm_100 cluster launch control).  The 16-byte response lands in
// shared memory at `resp16` (16-byte aligned) as transaction bytes on `bar`;
// the caller has armed `bar` with mbar_arrive_expect_tx(bar, 16).  A CTA
// whose request succeeds must run the cancelled CTA's work itself, which
// makes a grid of ordinary CTAs behave like persistent ones that take work
// in launch order.
__device__ __forceinline__ void clc_try_cancel(void* resp16, uint64_t* bar) {
  asm volatile(
      "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128"
      " [%0], [%1];" ::"r"(smem_u32(resp16)),
      "r"(smem_u32(bar))
      : "memory");
}

// blockIdx.x of the CTA a completed request cancelled, or -1 when the grid
// had no CTA left to cancel.
__device__ __forceinline__ int clc_result_x(const void* resp16) {
  uint32_t canceled, x = 0;
  asm volatile(
      "{\n\t.reg .b128 rsp;\n\t.reg .pred p;\n\t"
      "ld.shared.b128 rsp, [%2];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, rsp;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t"
      "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, rsp;\n\t}"
      : "=r"(canceled), "+r"(x)
      : "r"(smem_u32(resp16))
      : "memory");
  return canceled ? static_cast<int>(x) : -1;
}

// Work items of a persistent CTA (see clc_try_cancel).  Item 0 is the CTA's
// own blockIdx.x; item it >= 1 is the answer to the request the producer
// thread issued while it worked on item it - 1, kept in slot it & 1 of a
// two-slot ring (16-byte responses `resp`, barriers full[2] / empty[2]); the
// consumer warps release a slot through `empty` after reading it.

// Consumer side, called by all lanes of a warp.  Returns false when the
// wait gave up; idx < 0 means the grid has no work left.
__device__ __forceinline__ bool next_work_item(int it, int& idx, uint64_t* full, uint64_t* empty,
                                               const uint8_t* resp, volatile int* abort,
                                               const WaitCtl& ctl, int site) {
  if (it == 0) {
    idx = static_cast<int>(blockIdx.x);
    return true;
  }
  const int sl = it & 1;
  const bool w = mbar_wait(full + sl, static_cast<uint32_t>((it - 1) >> 1) & 1, abort, ctl, site);
  if (!__all_sync(0xffffffffu, w)) return false;
  idx = clc_result_x(resp + 16 * sl);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty + sl);
  return true;
}

// Producer side, called by all lanes of the producer warp: the answer for
// item it >= 1.
__device__ __forceinline__ bool producer_take_item(int it, int& idx, uint64_t* full,
                                                   const uint8_t* resp, volatile int* abort,
                                                   const WaitCtl& ctl, int site) {
  const int sl = it & 1;
  const bool w = mbar_wait(full + sl, static_cast<uint32_t>((it - 1) >> 1) & 1, abort, ctl, site);
  if (!__all_sync(0xffffffffu, w)) return false;
  idx = clc_result_x(resp + 16 * sl);
  return true;
}

// Producer side, called by all lanes of the producer warp: request item
// it + 1 into slot (it + 1) & 1 once the consumers have read that slot's
// previous answer; `leader` (one lane) issues it.  `pending` and
// `pending_par` record the request in flight (drained on abort).
__device__ __forceinline__ bool producer_request_item(int it, uint64_t* full, uint64_t* empty,
                                                      uint8_t* resp, volatile int* abort,
                                                      const WaitCtl& ctl, int site, bool leader,
                                                      int& pending, uint32_t& pending_par) {
  const int sl = (it + 1) & 1;
  const uint32_t u = static_cast<uint32_t>(it >> 1);
  if (u > 0) {
    const bool w = mbar_wait(empty + sl, (u - 1) & 1, abort, ctl, site);
    if (!__all_sync(0xffffffffu, w)) return false;
  }
  if (leader) {
    mbar_arrive_expect_tx(full + sl, 16);
    clc_try_cancel(resp + 16 * sl, full + sl);
  }
  __syncwarp();
  pending = sl;
  pending_par = u & 1;
  return true;
}

// Contiguous (untiled) bulk copy global -> shared, completion as transaction
// bytes on `bar`.  Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled store of a shared-memory box into global memory (rows and
// columns outside the tensor are not written); completion is tracked with
// bulk groups.  The box starts at a non-negative coordinate.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 16-byte store to shared memory.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 3-D tiled reduction (element-wise add, no multicast) of a shared-memory box
// into global memory; completion is tracked with bulk groups.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, const void* src, int x,
                                                  int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the shared-memory sources of all committed bulk groups are read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until all committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 32-byte store to global memory (the address 32-byte aligned): one whole
// L2 sector per thread.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Hint: bring the 128-byte line holding `p` into L1 (no register, no wait).
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Make generic-proxy writes to shared memory visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void fence_async_shared() {
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
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor as two 32-bit words.  The issuing thread
// builds each operand family's descriptor once and advances it per k-step
// or stage by adding the byte offset / 16 to the low word (the 14-bit start
// address field; shared addresses stay below 256 KB, so no carry leaves it).
// Keeping the per-MMA work to an add is what lets a single thread that shares
// its sub-partition with busy softmax warps keep the tensor core fed.
struct SDesc {
  uint32_t lo, hi;
};
// 128-byte-swizzled operand at shared address `saddr`.
//   K-major tile: rows of 64 bf16 (128 B), 8-row groups 1024 B apart (SBO);
//                 LBO unused (16).  A k-step of 16 elements advances 32 B.
//   MN-major tile: 64 MN-contiguous elements per 128-B row, one row per k;
//                 8-k groups SBO apart, 64-wide MN atoms LBO apart.
__device__ __forceinline__ SDesc sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  SDesc d;
  d.lo = ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
  d.hi = ((sbo >> 4) & 0x3FFFu) | (1u << 14) /* version (sm_100) */ | (2u << 29) /* 128B swizzle */;
  return d;
}
__device__ __forceinline__ SDesc operator+(SDesc d, uint32_t bytes) {
  d.lo += bytes >> 4;
  return d;
}

// D[tmem] (+)= A[smem] * B[smem]^T, one 16-deep k-step, bf16 in, fp32 acc.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, SDesc a, SDesc b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\t"
      "mov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a.lo), "r"(a.hi), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], A read from tensor memory (K-major).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, SDesc b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D,
// shape M x N (x16), operand majors (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                              // D format f32
         | (1u << 7)                            // A format bf16
         | (1u << 10)                           // B format bf16
         | (static_cast<uint32_t>(a_mn) << 15)  // A major
         | (static_cast<uint32_t>(b_mn) << 16)  // B major
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets
// columns [c, c+32) of lane (warp quarter * 32 + t).
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

// Warpgroup register re-allocation.  The block's register budget is fixed at
// launch (threads x registers per thread); every warpgroup of the block must
// execute one of these, and the shares must add up to at most that budget.
template <int R>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

// ------------------------------------------------------------ arithmetic

// f(std::integral_constant<int, 0>{}), ..., f(std::integral_constant<int, N - 1>{}):
// a loop whose index is a compile-time constant in the body.
template <int N, int I = 0, class F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (I < N) {
    f(std::integral_constant<int, I>{});
    static_for<N, I + 1>(f);
  }
}

// Largest of three values (one instruction on sm_100; like fmaxf, a NaN
// input is ignored in favour of the others).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest of N values (N a multiple of 8): eight independent chains of
// three-input maxima, so the reduction is N/2 instructions about N/16 deep.
template <int N>
__device__ __forceinline__ float row_max(const float (&s)[N]) {
  static_assert(N % 8 == 0 && N >= 16, "row_max wants a multiple of 8, at least 16");
  constexpr int kPairs = (N - 8) / 16;  // steps that fold two more values per chain
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = s[i];
#pragma unroll
  for (int k = 0; k < kPairs; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmax3(acc[i], s[8 + 16 * k + i], s[16 + 16 * k + i]);
#pragma unroll
  for (int c = 8 + 16 * kPairs; c < N; c += 8)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaxf(acc[i], s[c + i]);
  return fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]),
               fmaxf(acc[6], acc[7]));
}

// 2^x on the special-function unit (approximate, flush-to-zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two values on the FMA pipe (no special-function unit):
// 2^x = 2^n 2^f with n = round(x) (via the 1.5 * 2^23 shifter) and
// f = x - n in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose coefficients
// are the relative-error minimax fit on [-1/2, 1/2] computed by
// exact_io_aware_99_b200/fit_exp2.py (max relative error 7.5e-5); 2^n is
// added to the exponent field.  x is clamped to -126, so very negative
// arguments (and -inf) give about 1.2e-38 rather than 0: callers zero masked
// entries themselves.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kC0 = 0.9999280571937561f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.2426111251115799f, kC3 = 0.0551716685295105f;
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(kShift, kShift));
  const float2 n = __fadd2_rn(t, make_float2(-kShift, -kShift));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 p = __ffma2_rn(make_float2(kC3, kC3), f, make_float2(kC2, kC2));
  p = __ffma2_rn(p, f, make_float2(kC1, kC1));
  p = __ffma2_rn(p, f, make_float2(kC0, kC0));
  p.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  p.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return p;
}

// Pack two floats to bf16x2 (round to nearest even): `lo` in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Walks a set of tiles in increasing order, 32 tiles per word: `t.word(w)`
// returns the bits of tiles 32 w .. 32 w + 31 (computed by a converged warp,
// e.g. with a ballot), `t.n_t` the number of tiles.  Warp-uniform: every lane
// holds the same state.
struct TileCursor {
  int w = -1, nw;
  uint32_t bits = 0;
  __device__ explicit TileCursor(int n_t) : nw((n_t + 31) / 32) {}
  template <class Tiles>
  __device__ __forceinline__ int next(const Tiles& t) {
    while (bits == 0) {
      if (++w >= nw) return t.n_t;
      bits = t.word(w);
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1;
    return 32 * w + b;
  }
};

// One lane of a converged warp (elect.sync over the full mask).  The MMA
// issuers run their whole loop on all 32 lanes -- waits, fences and branches
// stay warp-uniform -- and only the elected lane issues tcgen05.mma/commit.
// Issuing from a lane-0 branch instead costs a quarter of the tensor rate
// once mbarrier waits sit between MMA groups (measured on B200: 659 vs 540
// cycles per 128x128x128 group).
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

}  // namespace fa
