// p·V for callers that cannot allocate device memory.
//
// packkv_pv_gemv takes a caller-allocated workspace for its split-K partial
// sums.  Some callers have no way to provide one: a runtime that reserves and
// plans all device memory once at start-up and forbids later allocations, a
// plain C or foreign-function host that has no device allocator to hand, or a
// decode loop that must not call cudaMalloc because it implicitly synchronises
// the device and stalls the other streams.  packkv_pv_gemv_noalloc runs the
// same kernels with the partials in a fixed scratch array that is part of the
// library image (PACKKV_PV_NOALLOC_SCRATCH_BYTES, 8 MiB of every GPU that
// loads the library, held until the process exits).  It allocates nothing.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "packkv.h"

namespace {

static __device__ __align__(256) unsigned char g_pv_scratch[PACKKV_PV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_pv_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pv_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

packkv_status packkv_pv_gemv_noalloc(const packkv_cache* cache, const float* p, int64_t ld_p, int32_t q_heads,
                                     float* out, void* stream) {
  const packkv_status st = packkv_cache_check(cache);
  if (st != PACKKV_OK) return st;
  if (cache->seq_blocks != nullptr || cache->block_table != nullptr) return PACKKV_ERR_UNSUPPORTED;
  if (q_heads < 1 || q_heads % cache->kv_heads != 0) return PACKKV_ERR_INVALID_ARG;
  const int g = q_heads / cache->kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return PACKKV_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)cache->n_blocks * PACKKV_BLOCK_TOKENS + cache->tail_len;
  if (!aligned16(p) || !aligned16(out) || ld_p < T || ld_p % 4 != 0) return PACKKV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    const size_t bytes = (size_t)cache->batch * q_heads * PACKKV_HEAD_DIM * sizeof(float);
    return cudaMemsetAsync(out, 0, bytes, s) == cudaSuccess ? PACKKV_OK : PACKKV_ERR_CUDA;
  }
  packkv::GemvArgs a{};
  a.arena = cache->v_arena;
  a.index = cache->v_index;
  a.tail = cache->v_tail;
  a.batch = cache->batch;
  a.kv_heads = cache->kv_heads;
  a.group = g;
  a.g_total = g;
  a.g_off = 0;
  a.max_blocks = cache->max_blocks;
  a.n_blocks = cache->n_blocks;
  a.tail_len = cache->tail_len;
  a.bits = (int)cache->fmt.bits;
  a.arena16 = cache->arena_bytes / 16;
  a.ctrl = cache->ctrl;
  a.items_per_bh = cache->n_blocks + (cache->tail_len > 0 ? 1 : 0);
  a.n_items = (long)cache->batch * cache->kv_heads * a.items_per_bh;
  a.p = p;
  a.ld = ld_p;
  a.out = out;
  size_t need = 0;
  if (packkv::pv_launch_workspace_bytes(a, &need) != cudaSuccess) return PACKKV_ERR_CUDA;
  if (need > PACKKV_PV_NOALLOC_SCRATCH_BYTES) return PACKKV_ERR_CAPACITY;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return PACKKV_ERR_CUDA;
  a.partials = reinterpret_cast<float*>(scratch);
  return packkv::launch_pv(a, nullptr, s) == cudaSuccess ? PACKKV_OK : PACKKV_ERR_CUDA;
}

}  // extern "C"
