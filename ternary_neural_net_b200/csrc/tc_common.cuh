// Device helpers shared by the tcgen05 kernels (not part of the ABI): shared-
// memory matrix descriptors, bounded mbarrier waits, TMA tile loads and
// tensor-memory loads.
#pragma once

#include <cstdint>

namespace bnn {
namespace tc {

constexpr uint64_t kWaitNs = 1000000000ull;  // a bounded mbarrier wait gives up after 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// groups 1024 bytes apart (rows of 128 bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address (16-byte units)
  d |= static_cast<uint64_t>(1) << 16;                 // leading-dimension offset (unused for this layout)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                 // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                 // 128-byte swizzle
  return d;
}

// One poll of an mbarrier phase, without suspending.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for an mbarrier phase.  polls == 0: polls for up to kWaitNs of
// wall time (%globaltimer, read every 64 polls); polls > 0: at most that many
// polls (the short bound of the diagnostic bnn_probe_wait_limit).  False when
// it ran out (counted in *errors, abort raised) or when another thread of the
// CTA raised the abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* errors, uint32_t polls = 0) {
  if (polls) {
    for (uint32_t it = 0; it < polls; ++it)
      if (mbar_try(bar, parity)) return true;
  } else {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try(bar, parity)) return true;
      if ((it & 63u) == 0) {
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) break;
      }
    }
  }
  *abort_flag = 1;
  atomicAdd(errors, 1u);
  return false;
}

// The same wait for threads that only wait (MMA issue, copies, epilogue):
// between polls the thread sleeps, leaving the issue slots of its SM
// sub-partition to the warps that compute.
__device__ __forceinline__ bool mbar_wait_idle(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               unsigned int* errors) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitNs) break;
    }
    __nanosleep(32);
  }
  *abort_flag = 1;
  atomicAdd(errors, 1u);
  return false;
}

// One poll with acquire semantics at cluster scope: the arrivals it observes
// may come from the other CTA of a cluster (see mbar_arrive_rank), whose
// shared-memory writes before its arrival are then visible here.
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait with cluster-scope acquire (same bounds and abort protocol).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  unsigned int* errors, uint32_t polls = 0) {
  if (polls) {
    for (uint32_t it = 0; it < polls; ++it)
      if (mbar_try_cluster(bar, parity)) return true;
  } else {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_cluster(bar, parity)) return true;
      if ((it & 63u) == 0) {
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) break;
      }
    }
  }
  *abort_flag = 1;
  atomicAdd(errors, 1u);
  return false;
}

// Arrive, with release semantics at cluster scope, on the mbarrier at the same
// shared-memory offset in CTA `rank` of the cluster (this CTA's own included).
__device__ __forceinline__ void mbar_arrive_rank(uint32_t bar, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(bar), "r"(rank));
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(remote) : "memory");
}

// Bounded wait that ignores the abort flag (the final drains).
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, unsigned int* errors) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63u) == 0 && global_ns() - t0 > kWaitNs) break;
  }
  atomicAdd(errors, 1u);
  return false;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// Named barrier 1 over the first `count` threads of the CTA (whole warps) that
// returns the AND of every participant's `pred`.
__device__ __forceinline__ bool producer_barrier_and(bool pred, int count) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.and.pred q, 1, %2, p;\nselp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(count)
      : "memory");
  return r != 0;
}

// Named barrier `id` over `count` threads (whole warps) returning the AND of
// every participant's `pred`.
__device__ __forceinline__ bool named_barrier_and(bool pred, int id, int count) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.and.pred q, %2, %3, p;\nselp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// 2-D tiled TMA load of one box into this CTA's shared memory (x = innermost
// element index, y = row), completing its bytes on the mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Arrives on the mbarrier once every tcgen05 operation this thread issued
// before it has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}

// 16 columns of this warp's 32 tensor-memory lanes (wait with tmem_wait_ld)
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
}

// 32 columns of this warp's 32 tensor-memory lanes (wait with tmem_wait_ld)
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

}  // namespace tc
}  // namespace bnn
