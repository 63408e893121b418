// Internal launch interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "packkv.h"

namespace packkv {

// Ragged batches (sequences of their own lengths) are described to the kernels by value,
// in the launch's parameter space: per sequence b, base[b] = its first item in the flat
// (sequence, head, item) list and tail[b] = its tail tokens (items of b: base[b+1] -
// base[b] = kv_heads * (blocks + (tail > 0))).  At most kMaxRaggedBatch sequences.
constexpr int kMaxRaggedBatch = PACKKV_RAGGED_MAX_BATCH;
struct RaggedPlan {
  int32_t base[kMaxRaggedBatch + 1];
  int32_t tail[kMaxRaggedBatch];
};
// The sequences an encode call touches, in order, and the logical block each starts at.
struct RaggedEncodePlan {
  int32_t seq[kMaxRaggedBatch];
  int32_t first_block[kMaxRaggedBatch];
};
// The tail position each sequence appends at (-1: the sequence takes no token).
struct RaggedAppendPlan {
  int32_t pos[kMaxRaggedBatch];
};

struct EncodeArgs {
  const uint16_t* k;  // [batch][heads][nb*128][128] fp16
  const uint16_t* v;
  int batch, heads, nb, n_old, max_blocks, bits, key_kind;
  int unit_mode;  // PACKKV_UNITS_*: unit base = smallest code, or 0
  uint32_t* k_index;
  uint32_t* v_index;
  uint8_t* k_arena;
  uint8_t* v_arena;
  uint64_t arena_bytes;
  uint8_t* perm;  // optional
  uint64_t* ctrl;
  // ragged calls: `batch` sequences of the plan (seq[s], first_block[s]); k, v rows are
  // (seq[s] * heads + h) * nb + i; block_table (optional, device) maps logical blocks
  const int32_t* block_table;
  bool ragged;
};

cudaError_t launch_encode(const EncodeArgs& a, const RaggedEncodePlan* plan, cudaStream_t stream);
cudaError_t launch_append(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail, int n_bh,
                          int pos, cudaStream_t stream);
// Ragged append: sequence b's token goes to tail position plan.pos[b] (none if negative).
cudaError_t launch_append_ragged(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail,
                                 int batch, int heads, const RaggedAppendPlan& plan, cudaStream_t stream);
size_t encode_smem_bytes();

// One decode GEMV over the packed cache (q·Kᵀ or p·V).
struct GemvArgs {
  const uint8_t* arena;
  const uint32_t* index;  // [batch][kv_heads][max_blocks][2]
  const uint16_t* tail;   // [batch][kv_heads][128][128] fp16
  int batch, kv_heads, group, max_blocks, n_blocks, tail_len, bits;
  int g_total, g_off;     // query heads per kv head, and the first one this launch serves
  uint64_t arena16;       // arena_bytes / 16
  uint64_t* ctrl;
  long n_items;           // batch*kv_heads*items_per_bh
  int items_per_bh;       // n_blocks + (tail_len > 0)
  int n_warps;            // logical warps sharing the items
  const int32_t* block_table;  // optional: physical block of (sequence, logical block)
  bool ragged;            // sequences of their own lengths (RaggedPlan passed with the launch)
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

cudaError_t launch_qk(GemvArgs a, const RaggedPlan* plan, cudaStream_t stream);
cudaError_t launch_pv(GemvArgs a, const RaggedPlan* plan, cudaStream_t stream);

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
  int g_total, g_off;       // query heads per kv head, and the first one this launch serves
  uint64_t arena16;         // arena_bytes / 16
  uint64_t* ctrl;
  long n_items;             // batch*kv_heads*items_per_bh
  int items_per_bh;         // n_blocks + (tail_len > 0)
  int n_warps;              // logical warps sharing the items
  const int32_t* block_table;  // optional: physical block of (sequence, logical block)
  bool ragged;              // sequences of their own lengths (RaggedPlan passed with the launch)
  const uint16_t* q;        // [batch][q_heads][128]
  float scale;
  float* out;               // [batch][q_heads][128]
  float* partials;          // [n_warps + batch*kv_heads][group][132]: sums [128], max, sum of exp
};

cudaError_t launch_attention(AttnArgs a, const RaggedPlan* plan, cudaStream_t stream);
size_t attention_workspace_bytes(int batch, int kv_heads, int group);

}  // namespace packkv
