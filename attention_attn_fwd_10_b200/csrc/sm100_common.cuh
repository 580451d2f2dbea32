// Blackwell (sm_100a) building blocks used by the attention kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (UMMA) descriptors,
// MMA issue/commit, TMEM allocation and TMEM <-> register moves, and the two
// exponentials (MUFU ex2 and the FMA-pipe cubic).
//
// Layout conventions shared by every kernel in this library:
// * global tensors are bf16 BSHD (D innermost); TMA views them as the 4-D
//   tensor (D, H, S, B) and fetches boxes of 64 x 1 x 128 x 1 elements, i.e.
//   128 rows of 128 bytes, with the 128-byte swizzle.  A 128 x D tile is D/64
//   such boxes, each 16 KiB and 1024-byte aligned in shared memory.
// * UMMA shared-memory descriptors describe those boxes either K-major (the
//   row is the contraction dim: Q and K in S = Q K^T) or MN-major (the row is
//   the contraction dim's partner: V in O += P V).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace attn {

// ----------------------------------------------------------------------------
// Status codes written by kernels to the library's device status word.
enum DeviceError : int {
  kDevOk = 0,
  kDevWaitTimeout = 5,  // matches ATTN_ERR_DEVICE_TIMEOUT
};

// ----------------------------------------------------------------------------
// Optional timeline, compiled in only with -DATTN_TIMELINE (a separate library,
// libattn_timeline.so; the default build has none of it): one chosen CTA records
// clock64() at fixed points of its pipeline, event ev of its block i, so a host
// tool can print the block cycle.  Events never change what a kernel computes.
#ifdef ATTN_TIMELINE
constexpr int kTimelineEvents = 16, kTimelineBlocks = 256;
__device__ long long g_timeline[kTimelineEvents][kTimelineBlocks];
__device__ long long g_timeline_t0;
__device__ int g_timeline_cta = -1;
#define ATTN_TL_ON() (static_cast<int>(blockIdx.x) == ::attn::g_timeline_cta)
#define ATTN_TL(on, ev, i)                                                        \
  do {                                                                            \
    if ((on) && (i) >= 0 && (i) < ::attn::kTimelineBlocks) ::attn::g_timeline[(ev)][(i)] = clock64(); \
  } while (0)
#define ATTN_TL_T0(on)                                            \
  do {                                                            \
    if ((on) && threadIdx.x == 0) ::attn::g_timeline_t0 = clock64(); \
  } while (0)
#else
#define ATTN_TL_ON() false
#define ATTN_TL(on, ev, i) \
  do {                     \
  } while (0)
#define ATTN_TL_T0(on) \
  do {                 \
  } while (0)
#endif

// ----------------------------------------------------------------------------
// Generic helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------------
// mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One arrival for the whole warp, after every lane has reached this point (and
// so after every lane's earlier writes and fences): 32x fewer shared-memory
// atomics on the barrier than an arrival per thread.
__device__ __forceinline__ void mbar_arrive_warp(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
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

// Shared control block for bounded waits: a CTA-wide abort flag in shared
// memory, the device status word, and the time limit of one wait.
struct WaitCtl {
  volatile int* abort_flag;  // shared memory
  int* status;               // global
  uint64_t limit_ns;
};

// Waits for the phase with the given parity to complete.  Gives up (returns
// false) when another thread of the CTA has already given up, or after
// ctl.limit_ns of wall time, in which case it raises the CTA's abort flag and
// records kDevWaitTimeout in the status word.  Never traps, never spins for ever.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*ctl.abort_flag) return false;
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicExch(ctl.status, kDevWaitTimeout);
        return false;
      }
    }
  }
}

// Waits until the global int at `sem` equals `want` (acquire at GPU scope), with
// the same bound and abort protocol as mbar_wait.
__device__ __forceinline__ bool sem_wait_eq(const int* sem, int want, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(sem) : "memory");
    if (v == want) return true;
    if ((it & 15u) == 0) {
      if (*ctl.abort_flag) return false;
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicExch(ctl.status, kDevWaitTimeout);
        return false;
      }
    }
  }
}

// Waits until the global int at `sem` is at least `want` (acquire at GPU scope),
// with the same bound and abort protocol as mbar_wait.
__device__ __forceinline__ bool sem_wait_ge(const int* sem, int want, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(sem) : "memory");
    if (v >= want) return true;
    if ((it & 15u) == 0) {
      if (*ctl.abort_flag) return false;
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicExch(ctl.status, kDevWaitTimeout);
        return false;
      }
    }
  }
}

// Adds 1 to the global int at `sem` with release semantics at GPU scope.
__device__ __forceinline__ void sem_release_add(int* sem) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(sem) : "memory");
}

// Orders global-memory accesses of the async proxy (TMA) against the generic proxy.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Same, but with a fixed limit and no abort check: used only while draining
// in-flight asynchronous work before a CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ----------------------------------------------------------------------------
// Cluster launch control: cancel the launch of a block (cluster of one) that has
// not started yet and take over its work.  The 16-byte response lands in shared
// memory and completes 16 transaction bytes on `bar`.  No further request may be
// made once a response has reported that nothing was cancelled.
__device__ __forceinline__ void clc_try_cancel(uint32_t resp_smem, uint32_t bar) {
  asm volatile(
      "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];" ::"r"(
          resp_smem),
      "r"(bar)
      : "memory");
}
// The x block index of the cancelled block, or -1 when nothing was cancelled.
__device__ __forceinline__ int clc_cancelled_block(uint32_t resp_smem) {
  uint32_t ok, x;
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b128 r;\n\t"
      "ld.shared.b128 r, [%2];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "clusterlaunchcontrol.query_cancel.get_first_ctaid.v4.b32.b128 {%1, _, _, _}, r;\n\t}"
      : "=r"(ok), "=r"(x)
      : "r"(resp_smem)
      : "memory");
  return ok ? static_cast<int>(x) : -1;
}

// ----------------------------------------------------------------------------
// Per-warpgroup register budgets (every warp of a warpgroup executes the same one).
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ----------------------------------------------------------------------------
// TMA: 4-D tiled load into shared memory, completion counted on an mbarrier.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// TMA: 4-D tiled reduce-add of a shared-memory tile into global memory (bulk group).
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of this thread's committed bulk groups have been read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tensor-core operand reads) before signalling their consumer.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM allocation
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

// ----------------------------------------------------------------------------
// UMMA descriptors
//
// Instruction descriptor for kind::f16 with bf16 A/B and an fp32 accumulator:
// bits [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
// bit 15 A major (0 = K), bit 16 B major (1 = MN), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, Blackwell version field:
// bits [0,14) start >> 4, [16,30) leading-dim byte offset >> 4, [32,46)
// stride-dim byte offset >> 4, [46,48) version = 1, [61,64) layout = 2 (SW128).
// K-major SW128: SBO = 1024 (next group of 8 rows), LBO unused (1).
// MN-major SW128: LBO = distance between 64-element column blocks, SBO = 1024
// (next group of 8 contraction rows).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// The same descriptor as two 32-bit halves.  The high half (SBO, version, layout)
// is a constant per operand kind; the low half is start >> 4 | (LBO >> 4) << 16, so
// the descriptor of start + off is the low half plus off >> 4 (shared-memory
// addresses are below 2^18: no carry leaves the 14-bit start field).
__host__ __device__ constexpr uint32_t sdesc_sw128_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B (type code 0 in
// the A / B format fields), both K-major, and an fp32 accumulator; the other
// fields as for kind::f16.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], 8-bit operands (K = 32 per instruction)
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// umma_ss / umma_ss_f8 / umma_ts / umma_ts_f8 with the shared-memory descriptors
// given as (low, high) halves, joined inside the instruction's asm.
__device__ __forceinline__ void umma_ss_h(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                          uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ss_f8_h(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                             uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_h(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_f8_h(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], b, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], 8-bit operands (K = 32 per instruction)
__device__ __forceinline__ void umma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// ----------------------------------------------------------------------------
// CTA pairs: clusters of two CTAs whose tensor cores execute one MMA together
// (cta_group::2).  The even CTA (rank 0) issues every MMA of the pair; an MMA
// of M rows takes rows [0, M/2) of A from rank 0 and [M/2, M) from rank 1, and
// the first / second half of B's N columns from rank 0 / rank 1, each at the
// same shared-memory (or tensor-memory) address in its own CTA, and leaves rank
// r's M/2 output rows (all N columns) in rank r's tensor memory.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Every thread of both CTAs (kernel start only: the pair is launched together).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of either CTA of the cluster (shared::cluster address).
// Default semantics (release at CTA scope), as the pair's hand-offs use: the data
// they order is tensor memory (tcgen05 fences around the arrival) or shared
// memory written by TMA and read by the tensor cores.
__device__ __forceinline__ void mbar_arrive_cl(uint32_t bar_cl) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cl) : "memory");
}
// Arrival that releases at cluster scope everything this thread has observed
// (after a CTA barrier: the whole CTA's earlier accesses to the other CTA), for
// the pair's exit handshake.  ~1.3k clk: not for per-block hand-offs.
__device__ __forceinline__ void mbar_arrive_cl_release(uint32_t bar_cl) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cl) : "memory");
}
// One mbar_arrive_cl for the whole warp, after every lane has reached this point.
__device__ __forceinline__ void mbar_arrive_cl_warp(uint32_t bar_cl) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cl(bar_cl);
}

__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait with acquire at cluster scope: for barriers that the other CTA of
// the pair arrives on (or commits to).
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*ctl.abort_flag) return false;
      if (globaltimer_ns() - t0 > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicExch(ctl.status, kDevWaitTimeout);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait_cl_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_cl(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from this
// CTA's shared memory into the shared memory of a cluster CTA (`dst_cl`); the
// transaction bytes complete on that CTA's mbarrier `bar_cl`.  Joins the issuing
// thread's current bulk group.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cl, uint32_t src, uint32_t bytes, uint32_t bar_cl) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cl),
               "r"(src), "r"(bytes), "r"(bar_cl)
               : "memory");
}

// 16-byte store into the shared memory of either CTA of the cluster.
__device__ __forceinline__ void st_shared_cl_v4(uint32_t addr_cl, uint4 v) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr_cl), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_shared_cl_u32(uint32_t addr_cl, uint32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr_cl), "r"(v) : "memory");
}

// Make this thread's generic-proxy writes to the shared memory of the cluster's
// CTAs visible to the async proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem_cl() {
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

// Tensor memory of a pair: one warp (same warp index) in each CTA executes these.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMAs (issued by rank 0), descriptors as (low, high) halves.
__device__ __forceinline__ void umma2_ss_h(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                           uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], a, b, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma2_ts_h(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], b, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on the mbarrier at shared::cluster address `bar_cl` (either CTA
// of the pair) when every pair MMA issued so far by this thread completes.
__device__ __forceinline__ void umma2_commit(uint32_t bar_cl) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cl)
               : "memory");
}

// High half of a 64-byte-swizzle descriptor (layout code 4): for MN-major
// operands whose rows are 32 bf16 (64 B); SBO = next group of 8 contraction rows.
__host__ __device__ constexpr uint32_t sdesc_sw64_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (4u << 29);
}

// ----------------------------------------------------------------------------
// TMEM <-> registers, shape 32x32b: the warp's 32 lanes (TMEM lanes 32*(warp%4)+i)
// each move 32 consecutive 32-bit columns.
#define ATTN_R8(a, o) "=r"(a[o + 0]), "=r"(a[o + 1]), "=r"(a[o + 2]), "=r"(a[o + 3]), \
                      "=r"(a[o + 4]), "=r"(a[o + 5]), "=r"(a[o + 6]), "=r"(a[o + 7])
#define ATTN_P8(a, o) "+r"(a[o + 0]), "+r"(a[o + 1]), "+r"(a[o + 2]), "+r"(a[o + 3]), \
                      "+r"(a[o + 4]), "+r"(a[o + 5]), "+r"(a[o + 6]), "+r"(a[o + 7])
#define ATTN_I8(a, o) "r"(a[o + 0]), "r"(a[o + 1]), "r"(a[o + 2]), "r"(a[o + 3]), \
                      "r"(a[o + 4]), "r"(a[o + 5]), "r"(a[o + 6]), "r"(a[o + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : ATTN_R8(r, 0), ATTN_R8(r, 8), ATTN_R8(r, 16), ATTN_R8(r, 24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : ATTN_R8(r, 0), ATTN_R8(r, 8)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait16(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : ATTN_P8(r, 0), ATTN_P8(r, 8) : : "memory");
}

// Wait for this thread's outstanding tcgen05.ld; the registers are threaded
// through the asm so no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : ATTN_P8(r, 0), ATTN_P8(r, 8), ATTN_P8(r, 16), ATTN_P8(r, 24)
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      ATTN_I8(r, 0), ATTN_I8(r, 8), ATTN_I8(r, 16), ATTN_I8(r, 24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      ATTN_I8(r, 0), ATTN_I8(r, 8)
      : "memory");
}

// Shape 16x256b, 4 repeats: lanes base + lane/4 and base + lane/4 + 8 of the
// 16-lane group at `taddr`, 32 columns.  r[4 k + 0..1] = row base + lane/4,
// columns 8 k + 2 (lane % 4) + {0, 1}; r[4 k + 2..3] = the same columns of row
// base + lane/4 + 8.
__device__ __forceinline__ void tmem_ld16x256_x4(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : ATTN_R8(r, 0), ATTN_R8(r, 8)
      : "r"(taddr));
}

// Shape 16x128b, 4 repeats: r[2 k + j] goes to row base + lane/4 + 8 j, column
// 4 k + lane % 4 (16 columns).
__device__ __forceinline__ void tmem_st16x128_x4(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), ATTN_I8(r, 0)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------------------
// Exponentials (base 2)

// Hardware unit (MUFU / SFU).  Flushes subnormals; ex2(-inf) = +0.
__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Software 2^x on the FMA pipe (FlashAttention-4's software exponential, as
// "AI Infra series ch. 6, GPU performance engineering (II)", section 7, item 1
// describes it: Cody-Waite range reduction plus a cubic).  With a base-2 input
// the reduction x = n + f is exact: n = floor(x) is obtained by one add in
// round-down mode against 1.5*2^23 (which leaves floor(x) in the low mantissa
// bits), f = x - n in [0, 1).  2^f is a cubic whose coefficients minimise the
// maximum relative error on [0, 1] (fit_exp2_poly.py; max rel. error 7.48e-5,
// 26x below the bf16 rounding of P).  2^n is applied by adding n to the
// exponent field: (t_bits << 23) equals n << 23 modulo 2^32 because the
// magic constant's own bits vanish under the shift.  Inputs are clamped at
// -126, so the exponent add never wraps into the sign bit; results below
// ~2^-125 are only guaranteed to be in [0, 2^-124).
constexpr float kExp2C0 = 9.999251962e-01f;  // 0x3f7ffb19
constexpr float kExp2C1 = 6.958335638e-01f;  // 0x3f322226
constexpr float kExp2C2 = 2.260671407e-01f;  // 0x3e677e25
constexpr float kExp2C3 = 7.802452892e-02f;  // 0x3d9fcb53


// ----------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot per two lanes of work)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The cubic above on a packed pair (two lanes of work per f32x2 instruction):
// clamp (two scalar max), floor via add.rm against 1.5*2^23, exact reduction,
// Horner in fma.f32x2, then the exponent-field add per lane.
__device__ __forceinline__ void exp2_poly_x2(uint64_t x2, float& e0, float& e1) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
  uint64_t t;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(t) : "l"(xc), "l"(magic));
  const uint64_t f = f2_sub(xc, f2_sub(t, magic));
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Four floats as e4m3 (round to nearest even, saturating at +-448) in one 32-bit
// word, a -> byte 0 ... d -> byte 3: four consecutive K elements of an 8-bit MMA
// operand in tensor memory.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Pack two floats into bf16x2 (round to nearest even): lo -> bits [0,16).
// Eight 32-bit words to global memory in one 256-bit store (sm_100); dst must be
// 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace attn
