// Device helpers shared by the kernels of libttt.so: status recording, bounded waits on
// mbarriers, and thin wrappers around the TMA / mbarrier / bulk-copy PTX of sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ttt {

// Status codes written by kernels (same values as ttt_status).
constexpr int kDevInvalidArg = 1;
constexpr int kDevUnsupported = 2;
constexpr int kDevTimeout = 5;
constexpr int kDevCheck = 6;

// Every spin-wait in this library gives up after a limit of %globaltimer nanoseconds (by
// default this many; a state can set its own), records TTT_ERR_TIMEOUT in the state's status
// word and lets the kernel wind down.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Where a kernel reports a failure, and how long each of its spin-waits may last.
struct DevStatus {
  int* word;             // status word (mapped host memory or device memory), or null
  uint64_t limit_ns;     // wait limit in %globaltimer nanoseconds
  int* site = nullptr;   // where the first failure happened (kSite* | detail), or null
};

// Sites of a wait that ran out: an mbarrier (detail: its shared-memory offset) or a progress
// counter in global memory (detail: the low bits of its word address).
constexpr int kSiteMbarrier = 0x10000;
constexpr int kSiteCounter = 0x20000;
// Argument checks that only the device can make, because the count they compare against lives
// on the device: the gate's token position would pass 2^31 − 1; the cache read's T is not the
// number of tokens gated since the reset (detail: the (sequence, head) index, low 16 bits).
constexpr int kSiteTokenLimit = 0x40000;
constexpr int kSiteCacheLength = 0x50000;

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ void record_status(const DevStatus& status, int code, int site = 0) {
  if (status.word != nullptr && atomicCAS(status.word, 0, code) == 0 && status.site != nullptr) *status.site = site;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// kCluster: acquire at cluster scope, for a barrier that another CTA of the cluster arrives on
// with release semantics (what that CTA wrote before arriving is then visible).
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  if constexpr (kCluster) {
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  }
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete. Returns false (after recording a timeout)
// if it has not completed within the wait limit, or at once if *abort is already set.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const DevStatus& status,
                                          volatile int* abort) {
  if (mbar_try_wait<kCluster>(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait<kCluster>(bar, parity)) return true;
    if ((++spins & 63u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer() - t0 > status.limit_ns) {
        record_status(status, kDevTimeout, kSiteMbarrier | (int)(smem_u32(bar) & 0xFFFFu));
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// ---- TMA (bulk tensor copies) ---------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset of element (row, col) of a bf16 tile with 128-byte rows stored with the
// TMA 128-byte swizzle (16-byte chunk index XOR row % 8). The tile base is 1024-aligned.
__device__ __forceinline__ uint32_t swz128_bf16(int row, int col) {
  const uint32_t byte = static_cast<uint32_t>(col) * 2u;
  return static_cast<uint32_t>(row) * 128u + ((((byte >> 4) ^ static_cast<uint32_t>(row & 7)) << 4) | (byte & 15u));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace ttt
