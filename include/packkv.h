/*
 * packkv.h — C ABI of the PackKV decode path for NVIDIA B200 (sm_100a).
 *
 * The operations follow the PackKV paper page ("PackKV: Reducing KV Cache
 * Memory Footprint through LLM-Aware Lossy Compression"):
 *   - abstract: a KV cache compressed so that it stays compatible with its
 *     dynamic growth during decoding, and decompression fused into the
 *     matrix-vector products;
 *   - Figure 1: each query dots every K vector, softmax, weighted sum of V;
 *   - Figure 2 and the TL;DR: quantize, reorder the quantized vectors (K and V
 *     bound together), bit-pack the integer codes along the channel direction;
 *     decompression inside the matrix-vector multiply, no write-back;
 *   - Figure 5: token-wise and channel-wise quantization granularity.
 * Every parameter the pages leave open is fixed by the packed-cache format, version 1.
 *
 * Conventions for every call:
 *   - Pointers named "device" are CUDA device pointers; all must be 16-byte
 *     aligned.  fp16 data is passed as uint16_t (IEEE binary16 bits).
 *   - The library never allocates, frees or synchronises memory, except
 *     packkv_get_status, which synchronises `stream` to read the status word.
 *     The caller owns every buffer.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     stream-ordered; host-side counters in packkv_cache are updated by the
 *     calls at enqueue time.
 *   - Errors found on the host are returned before anything is launched, and
 *     nothing is written.  Errors found on the device (arena full, non-finite
 *     input, corrupt index entry, a wait that gave up) set sticky bits in the
 *     cache's status word; packkv_get_status reads and clears them.  A block
 *     holding a NaN or Inf is still encoded, but its records are unspecified.
 *   - Thread safety: calls on one cache must be serialised by the caller.
 */
#ifndef PACKKV_H
#define PACKKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PACKKV_ABI_VERSION 3u
#define PACKKV_FORMAT_VERSION 1u
#define PACKKV_BLOCK_TOKENS 128
#define PACKKV_GROUP_TOKENS 32
#define PACKKV_HEAD_DIM 128
#define PACKKV_RAGGED_MAX_BATCH 2048  /* sequences of a ragged batch (see packkv_cache) */

typedef enum {
  PACKKV_OK = 0,
  PACKKV_ERR_INVALID_ARG = 1,  /* bad pointer, alignment, shape or counter */
  PACKKV_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. q_heads/kv_heads = 3) */
  PACKKV_ERR_CAPACITY = 3,     /* cache block table full (host) or arena full (device) */
  PACKKV_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  PACKKV_ERR_DEVICE = 5        /* device-detected error other than capacity */
} packkv_status;

/* Sticky device status bits (packkv_get_status). */
#define PACKKV_DEV_CAPACITY 0x1u   /* an encode did not fit in an arena; its blocks are invalid */
#define PACKKV_DEV_NONFINITE 0x2u  /* an encoded block held a NaN or Inf */
#define PACKKV_DEV_BAD_RECORD 0x4u /* a GEMV met an invalid index entry; its outputs are NaN/skipped */
#define PACKKV_DEV_TIMEOUT 0x8u    /* a kernel's bounded wait on an async copy gave up */

/* Reorder keys (packed-cache format v1, section 2). */
#define PACKKV_KEY_IDENTITY 0u
#define PACKKV_KEY_K_SUM 1u
#define PACKKV_KEY_KV_SUM 2u

/* How the encoder sizes a pack unit (packed-cache format v1, section 3; the PackKV
 * paper page, Figure 3: quantized codes concentrate on few values).  Both give format
 * v1 units (meta byte = base | width << 4) that every decode path reads alike:
 *   FOR:        frame of reference, base = the unit's smallest code, width = bit length
 *               of (largest - smallest);
 *   WIDTH_ONLY: base = 0, width = bit length of the largest code (for the ablation). */
#define PACKKV_UNITS_FOR 0u
#define PACKKV_UNITS_WIDTH_ONLY 1u

typedef struct {
  uint32_t version;      /* PACKKV_FORMAT_VERSION */
  uint32_t bits;         /* code width: 2, 3 or 4 */
  uint32_t block_tokens; /* 128 */
  uint32_t group_tokens; /* 32 */
  uint32_t head_dim;     /* 128 */
  uint32_t reorder_key;  /* PACKKV_KEY_* */
  uint32_t unit_mode;    /* PACKKV_UNITS_*: encoder only */
} packkv_format;

/*
 * The packed cache of one attention layer: plain data, every pointer owned by
 * the caller.  Zero ctrl[0..3] and set n_blocks = tail_len = 0 before first
 * use (packkv_cache_reset does both).
 *
 * Ragged batches and paged blocks (the visualisation page, "Read the caveat":
 * paging and multi-request scheduling).  With seq_blocks and seq_tail set, each
 * sequence b has its own length: seq_blocks[b] packed blocks and seq_tail[b]
 * (0..127) tail tokens.  Both are HOST arrays of `batch` int32 that the calls
 * read and advance at enqueue time, as they do n_blocks and tail_len for a
 * uniform batch (which must then stay 0); batch <= PACKKV_RAGGED_MAX_BATCH.
 * Scores and probabilities of sequence b are its first seq_blocks[b]*128 +
 * seq_tail[b] row entries; a sequence without tokens gets zero outputs.
 * With block_table set (uniform or ragged), logical block j of sequence b is the
 * physical block p = block_table[b*max_blocks + j] (device int32), whose records
 * the index entries at (p / max_blocks, head, p % max_blocks) name: sequences may
 * share blocks (a common prompt) and need not own contiguous index rows.  The
 * blocks an encode or append call creates must map to distinct physical blocks.
 */
typedef struct {
  packkv_format fmt;
  int32_t batch;       /* sequences */
  int32_t kv_heads;    /* KV heads per sequence */
  int32_t max_blocks;  /* block-table capacity per (sequence, head) */
  int32_t n_blocks;    /* host counter: packed blocks per (sequence, head), uniform over the batch */
  int32_t tail_len;    /* host counter: tokens in the uncompressed tail, 0..127 */
  int32_t reserved0;
  uint8_t* k_arena;    /* device, arena_bytes: K records (packed-cache format v1, section 4) */
  uint8_t* v_arena;    /* device, arena_bytes: V records */
  uint64_t arena_bytes;/* capacity of EACH arena; multiple of 16, at most 2^36 */
  uint32_t* k_index;   /* device u32 [batch][kv_heads][max_blocks][2] = {offset16, length16} */
  uint32_t* v_index;   /* device, same shape */
  uint16_t* k_tail;    /* device fp16 [batch][kv_heads][128][128], arrival order */
  uint16_t* v_tail;    /* device fp16, same shape */
  uint64_t* ctrl;      /* device u64[4]: K arena end (16-B units), V arena end, status bits, scratch */
  uint8_t* perm;       /* device, optional (NULL): u8 [batch][kv_heads][max_blocks][128],
                          perm[slot] = token index within the block (at the physical block) */
  int32_t* seq_blocks; /* host, optional (NULL = uniform batch): [batch] packed blocks per sequence */
  int32_t* seq_tail;   /* host, with seq_blocks: [batch] tail tokens per sequence */
  const int32_t* block_table; /* device, optional (NULL): [batch][max_blocks] physical blocks */
} packkv_cache;

/* ABI version and sizeof(packkv_cache), for bindings to check their mirror. */
uint32_t packkv_abi_version(void);
size_t packkv_cache_struct_size(void);
const char* packkv_status_string(packkv_status s);

/* Largest record of one block for `bits` (the raw record: 528 + 2048*bits bytes).
 * Returns 0 for unsupported bits. */
size_t packkv_record_bytes_max(uint32_t bits);

/* Workspace bytes packkv_pv_gemv needs for any n_blocks <= cache->max_blocks
 * with `q_heads` query heads (split-K partials).  packkv_qk_gemv needs none. */
size_t packkv_workspace_bytes(const packkv_cache* cache, int32_t q_heads);

/* Validates the struct (host-side checks only).  Nothing is launched. */
packkv_status packkv_cache_check(const packkv_cache* cache);

/* Zeroes ctrl[0..3] on `stream` and sets n_blocks = tail_len = 0. */
packkv_status packkv_cache_reset(packkv_cache* cache, void* stream);

/*
 * Encode n_blocks full blocks per (sequence, head) and append them to the cache
 * (quantize, joint token reorder, channel-direction bit-packing: packed-cache format v1,
 * sections 1-4; paper page Figures 2 and 5).
 *   k, v: device fp16 [batch][kv_heads][n_blocks*128][128], row-major.
 * Pack units are sized as cache->fmt.unit_mode says (PACKKV_UNITS_*).
 * Records go to the arenas in ascending (sequence, head, block) order.
 * Requires tail_len == 0 and n_blocks + cache->n_blocks <= max_blocks
 * (else PACKKV_ERR_INVALID_ARG / PACKKV_ERR_CAPACITY, nothing launched).
 * On success cache->n_blocks += n_blocks.  If an arena overflows on the device,
 * PACKKV_DEV_CAPACITY is set, the arena ends do not move and every new index
 * entry is marked invalid; records that fitted may have been written into the
 * free space past the old arena end.  One pass over the input: the records'
 * arena offsets come from a decoupled look-back over the new index entries
 * (which the call clears first) and ctrl[3] counts the call's blocks.
 * n_blocks == 0 is a no-op.
 * Ragged batch: every sequence gets n_blocks blocks after its own seq_blocks[b]
 * (every seq_tail[b] must be 0); seq_blocks[b] += n_blocks.
 */
packkv_status packkv_encode_block(packkv_cache* cache, const uint16_t* k, const uint16_t* v,
                                  int32_t n_blocks, void* stream);

/*
 * Append one token per (sequence, head) to the uncompressed tail (the cache's
 * dynamic growth, paper abstract).  k, v: device fp16 [batch][kv_heads][128].
 * When the tail reaches 128 tokens it is encoded as one block (as
 * packkv_encode_block) and tail_len returns to 0.
 * PACKKV_ERR_CAPACITY if the tail is full-to-be and the block table is full.
 * Ragged batch: every sequence appends at its own seq_tail[b]; the sequences whose
 * tail completes are encoded (in ascending order) into their next block.
 */
packkv_status packkv_append_token(packkv_cache* cache, const uint16_t* k, const uint16_t* v,
                                  void* stream);

/*
 * Ragged batch only: as packkv_append_token for the sequences with active[b] != 0
 * (host uint8 [batch]); the others take no token (k, v rows of those are not read).
 * This is how sequences of one batch come to differ in length (a request that
 * joins later, or one that has finished).  PACKKV_ERR_UNSUPPORTED for a uniform
 * batch.
 */
packkv_status packkv_append_token_masked(packkv_cache* cache, const uint16_t* k, const uint16_t* v,
                                         const uint8_t* active, void* stream);

/*
 * scores[b][hq][i] = scale * sum_c q[b][hq][c] * k_hat[b][hq/G][i][c]  (fp32 accumulate)
 * over the packed blocks in storage order, then the tail in arrival order
 * (packed-cache format v1, sections 6-7; paper page Figure 1, Figure 2 fused decompression).
 *   q:      device fp16 [batch][q_heads][128]; q_heads = G * kv_heads, G in {1,2,4,8,16,32,64}.
 *           G > 8 runs as G/8 launches of 8 query heads (the cache is read G/8 times).
 *           Several queries per kv head in one step (speculative decoding) are such a
 *           group: the S queries of the G heads of kv head h are rows h*S*G .. +S*G-1.
 *   scores: device fp32, row (b, hq) starts at (b*q_heads + hq) * ld_scores;
 *           ld_scores >= T = n_blocks*128 + tail_len (ragged: the longest sequence),
 *           multiple of 4.
 *   ws, ws_bytes: unused (may be NULL / 0).
 * The decompressed K is never written to memory.  T == 0 is a no-op.
 */
packkv_status packkv_qk_gemv(const packkv_cache* cache, const uint16_t* q, int32_t q_heads,
                             float scale, float* scores, int64_t ld_scores, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * out[b][hq][c] = sum_i p[b][hq][i] * v_hat[b][hq/G][i][c]  (fp32 accumulate)
 * with p in the same storage order as the scores.
 *   p:   device fp32, row (b, hq) at (b*q_heads + hq) * ld_p, ld_p >= T, multiple of 4.
 *   out: device fp32 [batch][q_heads][128].
 *   ws:  device, ws_bytes >= packkv_workspace_bytes(cache, q_heads): split-K
 *        partial sums over the sequence (no initialisation needed).  A second
 *        kernel adds them in a fixed order, so results are deterministic on a
 *        given GPU.  Two calls sharing one ws must not overlap in time.
 * With T == 0, out is set to zero.
 */
packkv_status packkv_pv_gemv(const packkv_cache* cache, const float* p, int64_t ld_p,
                             int32_t q_heads, float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * p·V without a caller-provided workspace.  (The PackKV pages have no
 * counterpart: this is a calling convention, not part of the method.)
 * For callers that cannot allocate device memory: runtimes that reserve all
 * device memory at start-up and forbid later allocations, hosts without a
 * device allocator to pass in, or decode loops that must not call cudaMalloc
 * because it synchronises the device.
 * Same arguments and result as packkv_pv_gemv minus ws/ws_bytes.  The split-K
 * partials live in a static device array of PACKKV_PV_NOALLOC_SCRATCH_BYTES
 * (8 MiB) that every GPU loading the library holds until the process exits;
 * the call allocates nothing.  It needs
 *     (W + batch*kv_heads) * G * 512 bytes,
 * W = the warps it launches = min(batch*kv_heads*items per pair, resident warps
 * of the p·V kernel: SMs x CTAs per SM x 4); e.g. on a B200 with 4-bit records
 * and G = 4 (2 CTAs per SM, W = 1184 once the cache has that many items) about
 * 2900 (sequence, kv head) pairs fit.  A call that needs more returns
 * PACKKV_ERR_CAPACITY without launching anything.
 * The first call on a device looks up the array's device address (a one-time
 * set-up, cached per device).
 * The cached address belongs to the device's current context: after a
 * cudaDeviceReset in the same process this entry point must not be used again.
 * All calls share the one array, and it keeps the last call's partials: calls
 * that overlap in time on the GPU race.  Nothing in it needs clearing (every
 * partial is written before it is read).  With T == 0, out is set to zero.
 * A ragged cache, one with a block table, or G above 8: PACKKV_ERR_UNSUPPORTED.
 */
#define PACKKV_PV_NOALLOC_SCRATCH_BYTES (8u << 20)
packkv_status packkv_pv_gemv_noalloc(const packkv_cache* cache, const float* p, int64_t ld_p,
                                     int32_t q_heads, float* out, void* stream);

/*
 * Decode attention over the packed cache in one pass (paper page, Figure 1: the
 * scores, the softmax and the weighted sum of values; Figure 2: decompression
 * inside the products):
 *   out[b][hq][c] = sum_i softmax_i(scale * q[b][hq]·k_hat[b][hq/G][i]) * v_hat[b][hq/G][i][c]
 * over every packed block and the tail.  The scores and probabilities never
 * reach global memory; the softmax is computed online (a running maximum and
 * sum of exponentials per warp), split over the sequence and merged with the
 * log-sum-exp rule by a second kernel in a fixed order (deterministic).
 *   q:   device fp16 [batch][q_heads][128]; q_heads = G * kv_heads, G in {1,2,4,8,16,32,64}
 *        (as for packkv_qk_gemv).
 *   out: device fp32 [batch][q_heads][128].
 *   ws:  device, ws_bytes >= packkv_attention_workspace_bytes(cache, q_heads)
 *        (no initialisation needed; two calls sharing ws must not overlap in time).
 * T == 0 (nothing to attend to) is PACKKV_ERR_INVALID_ARG for a uniform batch; in a
 * ragged batch a sequence without tokens gets zero outputs.  A record with an
 * invalid index entry sets PACKKV_DEV_BAD_RECORD and its tokens are left out.
 */
size_t packkv_attention_workspace_bytes(const packkv_cache* cache, int32_t q_heads);
packkv_status packkv_attention_decode(const packkv_cache* cache, const uint16_t* q, int32_t q_heads,
                                      float scale, float* out, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns PACKKV_OK if no device status bit is set,
 * else PACKKV_ERR_CAPACITY (capacity bit set) or PACKKV_ERR_DEVICE; stores
 * the bits in *bits_out (if not NULL) and clears them. */
packkv_status packkv_get_status(const packkv_cache* cache, void* stream, uint32_t* bits_out);

#ifdef __cplusplus
}
#endif

#endif /* PACKKV_H */
