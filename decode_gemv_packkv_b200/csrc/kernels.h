// Internal launch interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace packkv {

struct EncodeArgs {
  const uint16_t* k;  // [batch][heads][nb*128][128] fp16
  const uint16_t* v;
  int batch, heads, nb, n_old, max_blocks, bits, key_kind;
  uint32_t* k_index;
  uint32_t* v_index;
  uint8_t* k_arena;
  uint8_t* v_arena;
  uint64_t arena_bytes;
  uint8_t* perm;  // optional
  uint64_t* ctrl;
};

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t stream);
cudaError_t launch_append(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail, int n_bh,
                          int pos, cudaStream_t stream);
size_t encode_smem_bytes();

// One decode GEMV over the packed cache (q·Kᵀ or p·V).
struct GemvArgs {
  const uint8_t* arena;
  const uint32_t* index;  // [batch][kv_heads][max_blocks][2]
  const uint16_t* tail;   // [batch][kv_heads][128][128] fp16
  int batch, kv_heads, group, max_blocks, n_blocks, tail_len, bits;
  uint64_t arena16;       // arena_bytes / 16
  uint64_t* ctrl;
  long n_items;           // batch*kv_heads*items_per_bh
  int items_per_bh;       // n_blocks + (tail_len > 0)
  int n_warps;            // logical warps sharing the items
  // q·Kᵀ
  const uint16_t* q;      // [batch][q_heads][128]
  float* scores;          // row (b, hq) at (b*q_heads + hq) * ld
  long ld;
  float scale;
  // p·V
  const float* p;         // row (b, hq) at (b*q_heads + hq) * ld
  float* out;             // [batch][q_heads][128]
  float* partials;        // [n_warps + batch*kv_heads][group][128]
};

cudaError_t launch_qk(GemvArgs a, cudaStream_t stream);
cudaError_t launch_pv(GemvArgs a, cudaStream_t stream);

// Logical warps used by the GEMVs on the current device (an upper bound used
// for workspace sizing), and the workspace layout of p·V.
int gemv_max_warps();
size_t pv_workspace_bytes(int batch, int kv_heads, int group);
// Workspace bytes the launch of `a` by launch_pv would use (n_warps chosen as launch_pv does).
cudaError_t pv_launch_workspace_bytes(const GemvArgs& a, size_t* bytes);

// Fused decode attention over the packed cache: out = softmax(scale * q·Kᵀ) · V.
struct AttnArgs {
  const uint8_t* k_arena;
  const uint8_t* v_arena;
  const uint32_t* k_index;  // [batch][kv_heads][max_blocks][2]
  const uint32_t* v_index;
  const uint16_t* k_tail;   // [batch][kv_heads][128][128] fp16
  const uint16_t* v_tail;
  int batch, kv_heads, group, max_blocks, n_blocks, tail_len, bits;
  uint64_t arena16;         // arena_bytes / 16
  uint64_t* ctrl;
  long n_items;             // batch*kv_heads*items_per_bh
  int items_per_bh;         // n_blocks + (tail_len > 0)
  int n_warps;              // logical warps sharing the items
  const uint16_t* q;        // [batch][q_heads][128]
  float scale;
  float* out;               // [batch][q_heads][128]
  float* partials;          // [n_warps + batch*kv_heads][group][132]: sums [128], max, sum of exp
};

cudaError_t launch_attention(AttnArgs a, cudaStream_t stream);
size_t attention_workspace_bytes(int batch, int kv_heads, int group);

}  // namespace packkv
