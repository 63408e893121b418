// C ABI of the PackKV decode path: argument checks, host-side counters and
// kernel launches.  Declarations and the contract of every call: include/packkv.h.
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "packkv.h"

namespace {

using packkv::AttnArgs;
using packkv::EncodeArgs;
using packkv::GemvArgs;
using packkv::RaggedAppendPlan;
using packkv::RaggedEncodePlan;
using packkv::RaggedPlan;

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

packkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PACKKV_OK : PACKKV_ERR_CUDA; }

constexpr uint64_t kMaxArenaBytes = 0xFFFFFFFEull * 16ull;  // offsets fit u32, 0xFFFFFFFF = invalid

packkv_status check_cache(const packkv_cache* c) {
  if (c == nullptr) return PACKKV_ERR_INVALID_ARG;
  const packkv_format& f = c->fmt;
  if (f.version != PACKKV_FORMAT_VERSION || f.block_tokens != PACKKV_BLOCK_TOKENS ||
      f.group_tokens != PACKKV_GROUP_TOKENS || f.head_dim != PACKKV_HEAD_DIM)
    return PACKKV_ERR_UNSUPPORTED;
  if (f.bits < 2 || f.bits > 4) return PACKKV_ERR_UNSUPPORTED;
  if (f.reorder_key > PACKKV_KEY_KV_SUM) return PACKKV_ERR_UNSUPPORTED;
  if (f.unit_mode > PACKKV_UNITS_WIDTH_ONLY) return PACKKV_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->kv_heads < 1 || c->max_blocks < 1) return PACKKV_ERR_INVALID_ARG;
  if ((int64_t)c->batch * c->kv_heads > (1 << 24) || (int64_t)c->max_blocks > (1 << 24))
    return PACKKV_ERR_INVALID_ARG;
  if (c->n_blocks < 0 || c->n_blocks > c->max_blocks) return PACKKV_ERR_INVALID_ARG;
  if (c->tail_len < 0 || c->tail_len >= PACKKV_BLOCK_TOKENS) return PACKKV_ERR_INVALID_ARG;
  if (!aligned16(c->k_arena) || !aligned16(c->v_arena) || !aligned16(c->k_index) || !aligned16(c->v_index) ||
      !aligned16(c->k_tail) || !aligned16(c->v_tail) || !aligned16(c->ctrl))
    return PACKKV_ERR_INVALID_ARG;
  if (c->arena_bytes == 0 || (c->arena_bytes & 15u) != 0 || c->arena_bytes > kMaxArenaBytes)
    return PACKKV_ERR_INVALID_ARG;
  if ((c->seq_blocks == nullptr) != (c->seq_tail == nullptr)) return PACKKV_ERR_INVALID_ARG;
  if (c->block_table != nullptr && (reinterpret_cast<uintptr_t>(c->block_table) & 3u) != 0)
    return PACKKV_ERR_INVALID_ARG;
  if (c->seq_blocks != nullptr) {
    if (c->batch > PACKKV_RAGGED_MAX_BATCH) return PACKKV_ERR_UNSUPPORTED;
    if (c->n_blocks != 0 || c->tail_len != 0) return PACKKV_ERR_INVALID_ARG;
    for (int b = 0; b < c->batch; ++b)
      if (c->seq_blocks[b] < 0 || c->seq_blocks[b] > c->max_blocks || c->seq_tail[b] < 0 ||
          c->seq_tail[b] >= PACKKV_BLOCK_TOKENS)
        return PACKKV_ERR_INVALID_ARG;
  }
  return PACKKV_OK;
}

bool is_ragged(const packkv_cache* c) { return c->seq_blocks != nullptr; }

// Plans live in thread-local host storage: a launch copies its parameters when it is
// enqueued, so the storage is free again when the call returns.
RaggedPlan& plan_storage() {
  thread_local RaggedPlan p;
  return p;
}
RaggedEncodePlan& encode_plan_storage() {
  thread_local RaggedEncodePlan p;
  return p;
}
RaggedAppendPlan& append_plan_storage() {
  thread_local RaggedAppendPlan p;
  return p;
}

// The flat item list of a ragged cache: per sequence its first item and tail; returns
// the item count and the longest sequence (tokens).
RaggedPlan& build_plan(const packkv_cache* c, long* n_items, int64_t* t_max) {
  RaggedPlan& p = plan_storage();
  long acc = 0;
  int64_t tm = 0;
  for (int b = 0; b < c->batch; ++b) {
    p.base[b] = (int32_t)acc;
    p.tail[b] = c->seq_tail[b];
    acc += (long)(c->seq_blocks[b] + (c->seq_tail[b] > 0 ? 1 : 0)) * c->kv_heads;
    const int64_t tb = (int64_t)c->seq_blocks[b] * PACKKV_BLOCK_TOKENS + c->seq_tail[b];
    tm = tb > tm ? tb : tm;
  }
  p.base[c->batch] = (int32_t)acc;
  *n_items = acc;
  *t_max = tm;
  return p;
}

// Tokens of the longest sequence (uniform: every sequence).
int64_t max_tokens(const packkv_cache* c) {
  if (!is_ragged(c)) return (int64_t)c->n_blocks * PACKKV_BLOCK_TOKENS + c->tail_len;
  int64_t tm = 0;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t tb = (int64_t)c->seq_blocks[b] * PACKKV_BLOCK_TOKENS + c->seq_tail[b];
    tm = tb > tm ? tb : tm;
  }
  return tm;
}

EncodeArgs encode_args(const packkv_cache* c, const uint16_t* k, const uint16_t* v, int nb) {
  EncodeArgs a{};
  a.k = k;
  a.v = v;
  a.batch = c->batch;
  a.heads = c->kv_heads;
  a.nb = nb;
  a.n_old = c->n_blocks;
  a.max_blocks = c->max_blocks;
  a.bits = (int)c->fmt.bits;
  a.key_kind = (int)c->fmt.reorder_key;
  a.unit_mode = (int)c->fmt.unit_mode;
  a.k_index = c->k_index;
  a.v_index = c->v_index;
  a.k_arena = c->k_arena;
  a.v_arena = c->v_arena;
  a.arena_bytes = c->arena_bytes;
  a.perm = c->perm;
  a.ctrl = c->ctrl;
  a.block_table = c->block_table;
  a.ragged = false;
  return a;
}

// Query heads per kv head: 1, 2, 4 or 8 in one launch; 16, 32 or 64 (a wide group, or
// several queries per kv head, e.g. speculative decoding) in launches of 8 heads each.
bool group_ok(const packkv_cache* c, int32_t q_heads, int* group) {
  if (q_heads < 1 || q_heads % c->kv_heads != 0) return false;
  const int g = q_heads / c->kv_heads;
  *group = g;
  return g == 1 || g == 2 || g == 4 || g == 8 || g == 16 || g == 32 || g == 64;
}

constexpr int kMaxLaunchGroup = 8;  // query heads one launch serves
int launch_group(int g) { return g < kMaxLaunchGroup ? g : kMaxLaunchGroup; }

GemvArgs gemv_args(const packkv_cache* c, int group, const uint8_t* arena, const uint32_t* index,
                   const uint16_t* tail) {
  GemvArgs a{};
  a.arena = arena;
  a.index = index;
  a.tail = tail;
  a.batch = c->batch;
  a.kv_heads = c->kv_heads;
  a.group = launch_group(group);
  a.g_total = group;
  a.g_off = 0;
  a.max_blocks = c->max_blocks;
  a.n_blocks = c->n_blocks;
  a.tail_len = c->tail_len;
  a.bits = (int)c->fmt.bits;
  a.arena16 = c->arena_bytes / 16;
  a.ctrl = c->ctrl;
  a.items_per_bh = c->n_blocks + (c->tail_len > 0 ? 1 : 0);
  a.n_items = (long)c->batch * c->kv_heads * a.items_per_bh;
  a.block_table = c->block_table;
  a.ragged = is_ragged(c);
  return a;
}

// The ragged plan of a launch (nullptr for a uniform batch); sets a.n_items.
template <class A>
const RaggedPlan* launch_plan(const packkv_cache* c, A& a) {
  if (!is_ragged(c)) return nullptr;
  int64_t tm = 0;
  RaggedPlan& p = build_plan(c, &a.n_items, &tm);
  a.items_per_bh = 1;  // unused by ragged launches
  return &p;
}

}  // namespace

extern "C" {

uint32_t packkv_abi_version(void) { return PACKKV_ABI_VERSION; }

size_t packkv_cache_struct_size(void) { return sizeof(packkv_cache); }

const char* packkv_status_string(packkv_status s) {
  switch (s) {
    case PACKKV_OK: return "ok";
    case PACKKV_ERR_INVALID_ARG: return "invalid argument";
    case PACKKV_ERR_UNSUPPORTED: return "unsupported";
    case PACKKV_ERR_CAPACITY: return "capacity exceeded";
    case PACKKV_ERR_CUDA: return "CUDA error";
    case PACKKV_ERR_DEVICE: return "device-detected error";
  }
  return "unknown status";
}

size_t packkv_record_bytes_max(uint32_t bits) {
  if (bits < 2 || bits > 4) return 0;
  return (size_t)packkv::raw_record_bytes((int)bits);
}

size_t packkv_workspace_bytes(const packkv_cache* cache, int32_t q_heads) {
  if (check_cache(cache) != PACKKV_OK) return 0;
  int g = 0;
  if (!group_ok(cache, q_heads, &g)) return 0;
  return packkv::pv_workspace_bytes(cache->batch, cache->kv_heads, launch_group(g));
}

packkv_status packkv_cache_check(const packkv_cache* cache) { return check_cache(cache); }

packkv_status packkv_cache_reset(packkv_cache* cache, void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  const cudaError_t e = cudaMemsetAsync(cache->ctrl, 0, 4 * sizeof(uint64_t), as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  cache->n_blocks = 0;
  cache->tail_len = 0;
  if (is_ragged(cache))
    for (int b = 0; b < cache->batch; ++b) cache->seq_blocks[b] = cache->seq_tail[b] = 0;
  return PACKKV_OK;
}

packkv_status packkv_encode_block(packkv_cache* cache, const uint16_t* k, const uint16_t* v, int32_t n_blocks,
                                  void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  if (n_blocks < 0) return PACKKV_ERR_INVALID_ARG;
  if (!is_ragged(cache) && cache->tail_len != 0) return PACKKV_ERR_INVALID_ARG;
  if (n_blocks == 0) return PACKKV_OK;
  if (!aligned16(k) || !aligned16(v)) return PACKKV_ERR_INVALID_ARG;
  if ((int64_t)cache->batch * cache->kv_heads * n_blocks > 0x7fffffffLL) return PACKKV_ERR_INVALID_ARG;
  if (!is_ragged(cache)) {
    if ((int64_t)cache->n_blocks + n_blocks > cache->max_blocks) return PACKKV_ERR_CAPACITY;
    const cudaError_t e = packkv::launch_encode(encode_args(cache, k, v, n_blocks), nullptr, as_stream(stream));
    if (e != cudaSuccess) return PACKKV_ERR_CUDA;
    cache->n_blocks += n_blocks;
    return PACKKV_OK;
  }
  for (int b = 0; b < cache->batch; ++b) {
    if (cache->seq_tail[b] != 0) return PACKKV_ERR_INVALID_ARG;
    if ((int64_t)cache->seq_blocks[b] + n_blocks > cache->max_blocks) return PACKKV_ERR_CAPACITY;
  }
  RaggedEncodePlan& plan = encode_plan_storage();
  for (int b = 0; b < cache->batch; ++b) {
    plan.seq[b] = b;
    plan.first_block[b] = cache->seq_blocks[b];
  }
  EncodeArgs a = encode_args(cache, k, v, n_blocks);
  a.ragged = true;
  const cudaError_t e = packkv::launch_encode(a, &plan, as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  for (int b = 0; b < cache->batch; ++b) cache->seq_blocks[b] += n_blocks;
  return PACKKV_OK;
}

// One token for the sequences with active[b] (all if active is NULL) of a ragged cache.
packkv_status append_ragged(packkv_cache* cache, const uint16_t* k, const uint16_t* v, const uint8_t* active,
                            cudaStream_t stream) {
  RaggedAppendPlan& ap = append_plan_storage();
  RaggedEncodePlan& ep = encode_plan_storage();
  int n_done = 0;
  for (int b = 0; b < cache->batch; ++b) {
    const bool on = active == nullptr || active[b] != 0;
    ap.pos[b] = on ? cache->seq_tail[b] : -1;
    if (on && cache->seq_tail[b] + 1 == PACKKV_BLOCK_TOKENS) {
      if (cache->seq_blocks[b] >= cache->max_blocks) return PACKKV_ERR_CAPACITY;
      ep.seq[n_done] = b;
      ep.first_block[n_done] = cache->seq_blocks[b];
      ++n_done;
    }
  }
  cudaError_t e = packkv::launch_append_ragged(k, v, cache->k_tail, cache->v_tail, cache->batch, cache->kv_heads,
                                               ap, stream);
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  if (n_done > 0) {
    EncodeArgs a = encode_args(cache, cache->k_tail, cache->v_tail, 1);
    a.batch = n_done;
    a.ragged = true;
    e = packkv::launch_encode(a, &ep, stream);
    if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  }
  for (int b = 0; b < cache->batch; ++b) {
    if (ap.pos[b] < 0) continue;
    if (cache->seq_tail[b] + 1 == PACKKV_BLOCK_TOKENS) {
      cache->seq_blocks[b] += 1;
      cache->seq_tail[b] = 0;
    } else {
      cache->seq_tail[b] += 1;
    }
  }
  return PACKKV_OK;
}

packkv_status packkv_append_token(packkv_cache* cache, const uint16_t* k, const uint16_t* v, void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  if (!aligned16(k) || !aligned16(v)) return PACKKV_ERR_INVALID_ARG;
  if (is_ragged(cache)) return append_ragged(cache, k, v, nullptr, as_stream(stream));
  const bool completes = cache->tail_len + 1 == PACKKV_BLOCK_TOKENS;
  if (completes && cache->n_blocks >= cache->max_blocks) return PACKKV_ERR_CAPACITY;
  cudaError_t e = packkv::launch_append(k, v, cache->k_tail, cache->v_tail, cache->batch * cache->kv_heads,
                                        cache->tail_len, as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  if (!completes) {
    cache->tail_len += 1;
    return PACKKV_OK;
  }
  e = packkv::launch_encode(encode_args(cache, cache->k_tail, cache->v_tail, 1), nullptr, as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  cache->n_blocks += 1;
  cache->tail_len = 0;
  return PACKKV_OK;
}

packkv_status packkv_append_token_masked(packkv_cache* cache, const uint16_t* k, const uint16_t* v,
                                         const uint8_t* active, void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  if (!is_ragged(cache)) return PACKKV_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || active == nullptr) return PACKKV_ERR_INVALID_ARG;
  return append_ragged(cache, k, v, active, as_stream(stream));
}

packkv_status packkv_qk_gemv(const packkv_cache* cache, const uint16_t* q, int32_t q_heads, float scale,
                             float* scores, int64_t ld_scores, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  int g = 0;
  if (q_heads < 1 || q_heads % cache->kv_heads != 0) return PACKKV_ERR_INVALID_ARG;
  if (!group_ok(cache, q_heads, &g)) return PACKKV_ERR_UNSUPPORTED;
  const int64_t T = max_tokens(cache);
  if (!aligned16(q) || !aligned16(scores) || ld_scores < T || ld_scores % 4 != 0) return PACKKV_ERR_INVALID_ARG;
  if (T == 0) return PACKKV_OK;
  GemvArgs a = gemv_args(cache, g, cache->k_arena, cache->k_index, cache->k_tail);
  const RaggedPlan* plan = launch_plan(cache, a);
  a.q = q;
  a.scores = scores;
  a.ld = ld_scores;
  a.scale = scale;
  for (a.g_off = 0; a.g_off < g; a.g_off += a.group) {
    const cudaError_t e = packkv::launch_qk(a, plan, as_stream(stream));
    if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  }
  return PACKKV_OK;
}

packkv_status packkv_pv_gemv(const packkv_cache* cache, const float* p, int64_t ld_p, int32_t q_heads, float* out,
                             void* ws, size_t ws_bytes, void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  int g = 0;
  if (q_heads < 1 || q_heads % cache->kv_heads != 0) return PACKKV_ERR_INVALID_ARG;
  if (!group_ok(cache, q_heads, &g)) return PACKKV_ERR_UNSUPPORTED;
  const int64_t T = max_tokens(cache);
  if (!aligned16(p) || !aligned16(out) || ld_p < T || ld_p % 4 != 0) return PACKKV_ERR_INVALID_ARG;
  if (T == 0) {
    const size_t bytes = (size_t)cache->batch * q_heads * PACKKV_HEAD_DIM * sizeof(float);
    return cuda_status(cudaMemsetAsync(out, 0, bytes, as_stream(stream)));
  }
  const size_t need = packkv::pv_workspace_bytes(cache->batch, cache->kv_heads, launch_group(g));
  if (!aligned16(ws) || ws_bytes < need) return PACKKV_ERR_INVALID_ARG;
  GemvArgs a = gemv_args(cache, g, cache->v_arena, cache->v_index, cache->v_tail);
  const RaggedPlan* plan = launch_plan(cache, a);
  a.p = p;
  a.ld = ld_p;
  a.out = out;
  a.partials = reinterpret_cast<float*>(ws);
  for (a.g_off = 0; a.g_off < g; a.g_off += a.group) {  // launches of one stream: ws is reused in turn
    const cudaError_t e = packkv::launch_pv(a, plan, as_stream(stream));
    if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  }
  return PACKKV_OK;
}

size_t packkv_attention_workspace_bytes(const packkv_cache* cache, int32_t q_heads) {
  if (check_cache(cache) != PACKKV_OK) return 0;
  int g = 0;
  if (!group_ok(cache, q_heads, &g)) return 0;
  return packkv::attention_workspace_bytes(cache->batch, cache->kv_heads, launch_group(g));
}

packkv_status packkv_attention_decode(const packkv_cache* cache, const uint16_t* q, int32_t q_heads, float scale,
                                      float* out, void* ws, size_t ws_bytes, void* stream) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  int g = 0;
  if (q_heads < 1 || q_heads % cache->kv_heads != 0) return PACKKV_ERR_INVALID_ARG;
  if (!group_ok(cache, q_heads, &g)) return PACKKV_ERR_UNSUPPORTED;
  const int64_t T = max_tokens(cache);
  if ((T == 0 && !is_ragged(cache)) || !aligned16(q) || !aligned16(out)) return PACKKV_ERR_INVALID_ARG;
  const size_t need = packkv::attention_workspace_bytes(cache->batch, cache->kv_heads, launch_group(g));
  if (!aligned16(ws) || ws_bytes < need) return PACKKV_ERR_INVALID_ARG;
  AttnArgs a{};
  a.k_arena = cache->k_arena;
  a.v_arena = cache->v_arena;
  a.k_index = cache->k_index;
  a.v_index = cache->v_index;
  a.k_tail = cache->k_tail;
  a.v_tail = cache->v_tail;
  a.batch = cache->batch;
  a.kv_heads = cache->kv_heads;
  a.group = launch_group(g);
  a.g_total = g;
  a.max_blocks = cache->max_blocks;
  a.n_blocks = cache->n_blocks;
  a.tail_len = cache->tail_len;
  a.bits = (int)cache->fmt.bits;
  a.arena16 = cache->arena_bytes / 16;
  a.ctrl = cache->ctrl;
  a.items_per_bh = cache->n_blocks + (cache->tail_len > 0 ? 1 : 0);
  a.n_items = (long)cache->batch * cache->kv_heads * a.items_per_bh;
  a.block_table = cache->block_table;
  a.ragged = is_ragged(cache);
  const RaggedPlan* plan = launch_plan(cache, a);
  a.q = q;
  a.scale = scale;
  a.out = out;
  a.partials = reinterpret_cast<float*>(ws);
  for (a.g_off = 0; a.g_off < g; a.g_off += a.group) {
    const cudaError_t e = packkv::launch_attention(a, plan, as_stream(stream));
    if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  }
  return PACKKV_OK;
}

packkv_status packkv_get_status(const packkv_cache* cache, void* stream, uint32_t* bits_out) {
  const packkv_status st = check_cache(cache);
  if (st != PACKKV_OK) return st;
  uint64_t bits = 0;
  cudaError_t e = cudaMemcpyAsync(&bits, cache->ctrl + packkv::kCtrlStatus, sizeof(bits), cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  if (bits_out) *bits_out = (uint32_t)bits;
  if (bits == 0) return PACKKV_OK;
  e = cudaMemsetAsync(cache->ctrl + packkv::kCtrlStatus, 0, sizeof(uint64_t), as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return PACKKV_ERR_CUDA;
  return (bits & PACKKV_DEV_CAPACITY) ? PACKKV_ERR_CAPACITY : PACKKV_ERR_DEVICE;
}

}  // extern "C"
