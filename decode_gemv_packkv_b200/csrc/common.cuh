// Device-side helpers shared by the PackKV kernels (sm_100a).
//
// Record layout constants follow packed-cache format v1, section 4 (version 1).  The async
// copy helpers wrap the Hopper/Blackwell bulk-copy engine (cp.async.bulk with an
// mbarrier completion, never multicast) and the bounded mbarrier wait used by
// every kernel that stages records in shared memory.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "packkv.h"

namespace packkv {

constexpr int kBlockTokens = 128;
constexpr int kGroupTokens = 32;
constexpr int kHeadDim = 128;
constexpr int kGroups = 4;
constexpr int kHeaderBytes = 16;
constexpr int kParamOffset = 16;        // fp16 min[128] then fp16 scale[128]
constexpr int kMetaOffset = 528;        // compressed records only
constexpr int kRawWordOffset = 528;
constexpr int kPackedWordOffset = 1040;
constexpr uint32_t kRawFlag = 0x1u;
constexpr uint32_t kVFlag = 0x2u;

__host__ __device__ constexpr int raw_record_bytes(int bits) { return 528 + 2048 * bits; }

enum CtrlWord { kCtrlKEnd = 0, kCtrlVEnd = 1, kCtrlStatus = 2, kCtrlScratch = 3 };

__device__ __forceinline__ void set_status(uint64_t* ctrl, uint32_t bits) {
  atomicOr(reinterpret_cast<unsigned long long*>(ctrl + kCtrlStatus), (unsigned long long)bits);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier + bulk copy ---------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// Global -> shared bulk copy (no multicast).  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for phase `parity` of `bar` for at most ~1 s of wall time.  Returns
// false (and sets PACKKV_DEV_TIMEOUT) if it gave up; the caller then skips the
// staged data.  A copy that was issued always completes, so this never fires
// in a correct run; it only keeps a fault from turning into a hang.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t* ctrl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_ns() - start > 1000000000ull) {
      set_status(ctrl, PACKKV_DEV_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

}  // namespace packkv
