// Device-side helpers shared by the TQP MoE kernels (sm_100a only).
//
// Thin wrappers over the PTX of the Blackwell execution model: mbarriers with
// bounded waits, cp.async 16-byte copies, TMA 2-D tile loads, tcgen05 MMA /
// TMEM allocation / TMEM loads, the UMMA shared-memory and instruction
// descriptors, and bf16 helpers. Every spin on a barrier is bounded by a wall
// clock limit; on expiry it raises TQP_STATUS_TIMEOUT in the caller's status
// word and sets a CTA-wide abort flag so that all roles leave their loops.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "these kernels target sm_100a (B200) only"
#endif

namespace tqp {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per barrier wait (default)

// CTA-wide abort state in shared memory: the flag every role polls, and the
// limit of one barrier wait (kWaitLimitNs unless the launch asked for another).
struct Abort {
  int flag;
  int pad;
  unsigned long long limit_ns;
};

__device__ __forceinline__ void abort_init(Abort* ab, unsigned long long limit_ns) {
  ab->flag = 0;
  ab->limit_ns = limit_ns ? limit_ns : kWaitLimitNs;
}

__device__ __forceinline__ bool aborted(const Abort* ab) { return *reinterpret_cast<const volatile int*>(&ab->flag) != 0; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_status(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, with acquire at cluster scope: for barriers that also take
// arrivals from the other CTA of a pair.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity. Returns false (and sets the
// CTA abort flag and the timeout status bit) when the CTA's wait limit expires
// or another role has already aborted. kSleep > 0 backs off with nanosleep
// between polls, for waiters off the critical path (they then leave issue
// slots to the dequantising warps).
template <int kSleep = 0, bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Abort* ab, int32_t* status) {
  const uint32_t addr = smem_u32(bar);
  auto try_wait = [&]() { return kCluster ? mbar_try_wait_cluster(addr, parity) : mbar_try_wait(addr, parity); };
  if (try_wait()) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t limit = ab->limit_ns;
  // the clock is read every 64 polls, or every poll under a short test limit
  const uint32_t every = limit < 1000000ull ? 0u : 63u;
  uint32_t spins = 0;
  while (true) {
    if (try_wait()) return true;
    if (kSleep > 0) __nanosleep(kSleep);
    if (((++spins) & every) == 0u) {
      if (aborted(ab)) return false;
      if (globaltimer() - t0 > limit) {
        *reinterpret_cast<volatile int*>(&ab->flag) = 1;
        raise_status(status, TQP_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: every lane polls (measured faster than one polling
// lane with a broadcast), and the result is the same for the whole warp.
template <int kSleep = 0, bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, Abort* ab, int32_t* status) {
  return __all_sync(0xFFFFFFFFu, mbar_wait<kSleep, kCluster>(bar, parity, ab, status));
}

// One arrival for the whole warp, after every lane's preceding accesses.
__device__ __forceinline__ void mbar_arrive_warp(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Drain wait on the abort path: waits for the phase regardless of the abort
// flag, but no longer than limit_ns, so that asynchronous work issued before
// the abort (a TMA fill, committed MMAs) has finished before the CTA releases
// its shared and tensor memory. A phase that also needs arrivals that will
// never come (the other roles left their loops) just runs out.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns = 1000000ull) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(addr, parity)) {
    if (globaltimer() - t0 > limit_ns) return;
  }
}

// The TMA fills one thread has issued into a ring of barriers bar[0..N), so
// that on the abort path every fill still in flight is waited for, not only
// the last one (a fill landing after the CTA exits would write shared memory
// that the next CTA on the SM owns).
struct PendingFills {
  uint32_t mask = 0;     // stages with at least one issued fill
  uint32_t parity = 0;   // bit s: phase parity of the last fill of stage s
  __device__ __forceinline__ void issued(int stage, uint32_t ph) {
    mask |= 1u << stage;
    parity = (parity & ~(1u << stage)) | ((ph & 1u) << stage);
  }
  __device__ __forceinline__ void drain(uint64_t* bar0) const {
    for (int s = 0; s < 32; ++s)
      if (mask & (1u << s)) mbar_drain(bar0 + s, (parity >> s) & 1u);
  }
};

// ----------------------------------------------------------------------------
// async copies
// ----------------------------------------------------------------------------

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte global->shared copy; src_bytes < 16 zero-fills the rest (0 = all zeros).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

// Arrive on the barrier once every cp.async issued so far by this thread has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Completion of a thread's cp.async stages, made visible to the tensor cores.
// Each stage's copies form one commit group; the arrival on a stage's "full"
// barrier is delayed by kLag stages, after cp.async.wait_group has confirmed
// the group landed and fence.proxy.async has published the generic-proxy
// writes to the async proxy. kLag must be smaller than the ring depth.
template <int kLag>
struct CpAsyncLagArrive {
  uint64_t* pend[kLag + 1];
  int n = 0;
  __device__ __forceinline__ void stage_done(uint64_t* full_bar) {
    cp_async_commit();
    pend[n++] = full_bar;
    if (n > kLag) {
      cp_async_wait_group<kLag>();
      fence_proxy_async_smem();
      mbar_arrive(pend[0]);
#pragma unroll
      for (int i = 0; i < kLag; ++i) pend[i] = pend[i + 1];
      --n;
    }
  }
  __device__ __forceinline__ void flush() {
    cp_async_wait_all();
    fence_proxy_async_smem();
    for (int i = 0; i < n; ++i) mbar_arrive(pend[i]);
    n = 0;
  }
};

// TMA 2-D tile load (no multicast) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Hint: bring the 128-byte line holding p into L2.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05 (TMEM + UMMA)
// ----------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation, one CTA.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 inputs, fp32 accumulation, one CTA. A is
// M=128 lanes x K: each 32-bit column holds two consecutive K elements (the lower
// K index in the low half); a K step of 16 spans 8 columns.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ----------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs sharing one tcgen05.mma of M = 256)
// ----------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of this CTA's shared variable at `saddr` in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Arrive on a barrier of a CTA of this cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA 2-D tile load (no multicast) into this CTA's shared memory whose byte
// count completes on a barrier of the CTA pair (cta_group::2): `bar_cluster` is
// a shared::cluster address, here the even CTA's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// Every thread of both CTAs of the cluster (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Tensor memory of a CTA pair: both CTAs' allocating warps (the same warp index)
// allocate, relinquish and free together.
__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T across a CTA pair (M = 256): issued by one
// thread of the even CTA; each CTA holds 128 rows of A (TMEM, same address),
// half of B's N rows (shared memory, same offset) and its 128 x N quarter of D.
__device__ __forceinline__ void umma2_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once all
// previously issued pair MMAs of this thread completed.
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(uint16_t(3))
      : "memory");
}

// Arrive on the barrier when all previously issued tcgen05.mma of this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Instruction descriptor: kind::f16, A = B = fp16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Instruction descriptor: kind::f16, A = B = fp16, D = f32, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_f16_bmn(int M, int N) {
  return (1u << 4) | (1u << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory descriptor of an MN-major, 128B-swizzled 16-bit tile: 64 MN
// elements (128 B) per K row, 8 K rows per 1024-byte atom (SBO = 1024 B between
// atoms along K), 64-element MN columns `lbo` bytes apart (LBO). A K step of 16
// advances the start by 2048 B.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t((saddr & 0x3FFFF) >> 4)) | (uint64_t(lbo >> 4) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Shared-memory descriptor for a K-major, 128-byte-swizzled bf16 tile: rows of
// 64 elements (128 B), 8-row atoms of 1024 B stacked along M/N. The tile base
// must be 1024-byte aligned; a K sub-step of 16 elements advances the start by 32 B.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  return (uint64_t((saddr & 0x3FFFF) >> 4)) | (uint64_t(16 >> 4) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  // the wait names the destination registers so that no use is hoisted above it
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 / 16 consecutive 32-bit columns of this thread's TMEM lane, from registers.
// tmem_wait_st() must follow before the values are published to another thread.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// As tmem_st16, 4 columns.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3])
               : "memory");
}

// As tmem_st16, 8 columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------------------------------
// bf16
// ----------------------------------------------------------------------------

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return uint32_t(f32_to_bf16(lo)) | (uint32_t(f32_to_bf16(hi)) << 16);
}

// ----------------------------------------------------------------------------
// stream format of the additive coupling
// ----------------------------------------------------------------------------
// The coupling's streams are fp32 multiples of 2^-kStreamGridBits of magnitude
// below kStreamMax. Such a value has at most 24 significant bits, so the sum or
// difference of two of them is exact in fp32 while it stays below kStreamMax:
// the inverse's subtraction then returns the forward's input bit for bit, at
// any depth. Every bf16 value of magnitude 2^-9 or more lies on the grid; a
// smaller one moves by at most 2^-17 and stays a bf16 value.
constexpr int kStreamGridBits = 16;
constexpr float kStreamScale = float(1 << kStreamGridBits);
constexpr float kStreamMax = float(1 << (24 - kStreamGridBits));

__device__ __forceinline__ float to_stream_grid(float v) { return rintf(v * kStreamScale) * (1.0f / kStreamScale); }

// ----------------------------------------------------------------------------
// fp16 (operand type of the expert contractions)
// ----------------------------------------------------------------------------

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  return uint32_t(__half_as_ushort(__float2half_rn(lo))) | (uint32_t(__half_as_ushort(__float2half_rn(hi))) << 16);
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// bf16 bits -> fp16 bits, rounding to nearest even. Where the value is an fp16
// normal number it is exact (8 significant bits fit in 11) and done with integer
// arithmetic alone, by re-biasing the exponent from 127 to 15; zeros keep their
// sign; everything else (fp16 subnormals, overflow, inf, nan) takes the
// hardware conversion. Keeping the common case off the conversion pipe matters
// where that pipe is busy with transcendentals in other warps.
__device__ __forceinline__ uint32_t bf16_to_f16_bits(uint32_t b) {
  const uint32_t mag = b & 0x7FFFu;
  if ((mag >> 7) - 113u <= 29u) return (b & 0x8000u) | ((mag << 3) - (112u << 10));
  if (mag == 0u) return b & 0x8000u;
  return __half_as_ushort(__float2half_rn(__uint_as_float(b << 16)));
}

// As bf16_to_f16_bits, and sets `overflow` when the value does not fit fp16:
// a magnitude of 2^16 or more (bf16 values below that fit, with their 8
// significant bits), inf or nan. The check runs on the slow path only.
__device__ __forceinline__ uint32_t bf16_to_f16_bits_chk(uint32_t b, bool& overflow) {
  const uint32_t mag = b & 0x7FFFu;
  if ((mag >> 7) - 113u <= 29u) return (b & 0x8000u) | ((mag << 3) - (112u << 10));
  if (mag == 0u) return b & 0x8000u;
  overflow |= (mag >> 7) > 127u + 15u;
  return __half_as_ushort(__float2half_rn(__uint_as_float(b << 16)));
}

// 8 bf16 values (one 16-byte chunk) -> 8 fp16 values (exact within fp16 range).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = bf16_to_f16_bits(w[i] & 0xFFFFu) | (bf16_to_f16_bits(w[i] >> 16) << 16);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// As bf16x8_to_f16x8, setting `overflow` for any value that does not fit fp16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8_chk(uint4 v, bool& overflow) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = bf16_to_f16_bits_chk(w[i] & 0xFFFFu, overflow) | (bf16_to_f16_bits_chk(w[i] >> 16, overflow) << 16);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Nonzero when either fp16 half of the pair is inf or nan (exponent field all ones).
__device__ __forceinline__ uint32_t f16x2_nonfinite(uint32_t w) { return __vcmpeq2(w & 0x7C007C00u, 0x7C007C00u); }

// Byte offset of 16-byte chunk c (0..7) of row r inside a K-major SW128 tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t c) {
  return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

}  // namespace tqp
