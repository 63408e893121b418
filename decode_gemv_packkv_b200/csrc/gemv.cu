// Fused decompression + matrix-vector products over the packed cache
// (PackKV paper page, Figure 2 "computation-aware decompression + matrix-vector
// multiplication", TL;DR: decompression integrated into the GEMV with no
// write-back of decompressed data; Figure 1: the two decode products).
//
//   q·Kᵀ : scores[b,hq,i] = scale * sum_c q[b,hq,c] * k_hat[b,h,i,c]
//   p·V  : out[b,hq,c]    = sum_i p[b,hq,i] * v_hat[b,h,i,c]
//
// Design (sm_100a):
//  * Work = a flat list of items: for every (sequence, kv-head) its packed blocks
//    then, if present, its fp16 tail.  Each warp owns a contiguous range of
//    items (balanced to one item), so one packed-tile read serves all G query
//    heads of the kv head and neighbouring warps stream neighbouring records.
//  * Each warp runs its own STAGES-deep pipeline of shared-memory stages filled
//    by the bulk-copy engine (cp.async.bulk + mbarrier complete_tx; never
//    multicast).  A raw record is copied as a header/params piece plus 8 or 16
//    chunks at a padded pitch, so that the lanes' 32-bit reads of packed words
//    fall in distinct banks.  A compressed record is copied in one piece.
//  * Dequantization is folded out of the inner loop: k_hat = mn_c + s_c*(base+off)
//    gives score = scale*(sum_c q_c mn_c + sum_c (q_c s_c) base + sum_c (q_c s_c) off);
//    v_hat = mn_r + s_r*(base+off) gives out_c = sum_r p_r mn_r + sum_r (p_r s_r)(base+off).
//    The inner loop is one LOP3 (mask | 0x4B000000: the field becomes the low
//    mantissa bits of 2^23 + field*2^k), one FADD (removes 2^23 exactly) and one
//    FFMA per element and query head.  The power of two 2^k of each field
//    position is undone once per token (q·Kᵀ) or folded into p (p·V).
//  * q·Kᵀ: lanes split (group, token word, channel range); each lane keeps fp32
//    accumulators for 8 or 16 tokens and a 2- or 4-way shuffle sum finishes.
//  * p·V: lane = channel; a warp sums its item range into per-channel fp32
//    partials and writes them to the workspace at every (sequence, head)
//    boundary (split-K over the sequence); a second-pass kernel, launched as a
//    programmatic dependent so its launch overlaps the first, adds the partials
//    of each (sequence, head) in warp order: deterministic.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "kernels.h"

namespace packkv {

namespace {

#ifndef PACKKV_WARPS_PER_CTA
#define PACKKV_WARPS_PER_CTA 4
#endif
constexpr int kWarpsPerCta = PACKKV_WARPS_PER_CTA;
#ifndef PACKKV_WARP_SMEM_KB
#define PACKKV_WARP_SMEM_KB 10  // shared memory per warp: one stage, five CTAs of 4 warps per SM
#endif
constexpr int kWarpSmemBudget = PACKKV_WARP_SMEM_KB * 1024;
constexpr uint32_t kMagicBits = 0x4B000000u;
constexpr float kMagic = 8388608.0f;

enum ItemKind : int { kKindRaw = 0, kKindPacked = 1, kKindInvalid = 2, kKindTail = 3 };

__device__ __forceinline__ float mag(uint32_t field_bits) {
  return __uint_as_float(field_bits | kMagicBits) - kMagic;
}

// (w & mask) | 0x4B000000 in one LOP3: the field lands in the low mantissa bits of 2^23.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t fld(uint32_t w) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(kMagicBits));
  return d;
}

// Two magic-number fields -> their exact values, with one packed FP32 add.
__device__ __forceinline__ float2 pairf(uint32_t a, uint32_t b) {
  return __fadd2_rn(make_float2(__uint_as_float(a), __uint_as_float(b)), make_float2(-kMagic, -kMagic));
}

// Field position exponents of the in-register decode (value = field * 2^sig).
__host__ __device__ constexpr int sig4(int i) { return i <= 4 ? 4 * i : 4 * i - 12; }
__host__ __device__ constexpr int sig2(int i) { return i <= 10 ? 2 * i : 2 * i - 12; }
__host__ __device__ constexpr float pow2(int e) {
  return e >= 0 ? float(1u << e) : 1.0f / float(1u << (-e));
}
// 2^e for a run-time e in [-126, 127], from the exponent bits (no division)
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// 8 nibbles of a 4-bit slice word as 4 pairs: v[p] = (field_2p * 2^sig4(2p), field_2p+1 * 2^sig4(2p+1))
__device__ __forceinline__ void dec4(uint32_t w, float2 (&v)[4]) {
  const uint32_t h = w >> 12;
  v[0] = pairf(fld<0xFu>(w), fld<0xF0u>(w));
  v[1] = pairf(fld<0xF00u>(w), fld<0xF000u>(w));
  v[2] = pairf(fld<0xF0000u>(w), fld<0xF00u>(h));
  v[3] = pairf(fld<0xF000u>(h), fld<0xF0000u>(h));
}

template <int I>
__device__ __forceinline__ uint32_t fld2(uint32_t w, uint32_t h) {
  if constexpr (I <= 10)
    return fld<(3u << (2 * I))>(w);
  else
    return fld<(3u << (2 * I - 12))>(h);
}

// 16 two-bit fields of a 2-bit slice word as 8 pairs: field_i * 2^sig2(i)
__device__ __forceinline__ void dec2(uint32_t w, float2 (&v)[8]) {
  const uint32_t h = w >> 12;
  v[0] = pairf(fld2<0>(w, h), fld2<1>(w, h));
  v[1] = pairf(fld2<2>(w, h), fld2<3>(w, h));
  v[2] = pairf(fld2<4>(w, h), fld2<5>(w, h));
  v[3] = pairf(fld2<6>(w, h), fld2<7>(w, h));
  v[4] = pairf(fld2<8>(w, h), fld2<9>(w, h));
  v[5] = pairf(fld2<10>(w, h), fld2<11>(w, h));
  v[6] = pairf(fld2<12>(w, h), fld2<13>(w, h));
  v[7] = pairf(fld2<14>(w, h), fld2<15>(w, h));
}

// 3-bit raw unit, 16 tokens: 2-bit slice word w2 plus the 16 slice-1 bits at bits 0..15 of x.
// v[p] = (field2 + 4*bit) * 2^sig2, merged with one exact packed FMA per pair.
__device__ __forceinline__ void dec3(uint32_t w2, uint32_t x, float2 (&v)[8]) {
  dec2(w2, v);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int i = 2 * p;
    const float2 b = pairf(x & (1u << i) | kMagicBits, x & (2u << i) | kMagicBits);
    v[p] = __ffma2_rn(b, make_float2(pow2(sig2(i) - i + 2), pow2(sig2(i + 1) - i + 1)), v[p]);
  }
}

template <int BITS>
struct RawLayout;
template <>
struct RawLayout<4> {
  static constexpr int kChunks = 8, kChunkBytes = 1024;
};
template <>
struct RawLayout<3> {
  static constexpr int kChunks = 16, kChunkBytes = 384;
};
template <>
struct RawLayout<2> {
  static constexpr int kChunks = 16, kChunkBytes = 256;
};

template <int BITS, int G, bool PV>
struct Cfg {
  static constexpr int kChunks = RawLayout<BITS>::kChunks;
  static constexpr int kChunkBytes = RawLayout<BITS>::kChunkBytes;
  static constexpr int kPitch = kChunkBytes + 16;
  static constexpr int kChunksPerGroup = kChunks / 4;
  static constexpr int kChanPerChunk = 128 / kChunksPerGroup;  // 64 (b=4) or 32
  static constexpr int kRecBytes = raw_record_bytes(BITS);
  // b = 3 raw records are staged in padded chunks (bank-conflict-free CUDA-core decode);
  // b = 2 / 4 raw records are already in fragment order and are staged in one piece
  static constexpr bool kChunked = BITS == 3;
  static constexpr int kStageRec = kChunked ? 528 + kChunks * kPitch : kRecBytes;  // >= every record
  static constexpr int kStageBytes = kStageRec + (PV ? 512 * G : 0);
  static constexpr int kNT = (2 * G + 7) / 8;                  // MMA n-tiles: columns (head, hi/lo)
  static constexpr int kBTabBytes = 8 * (64 * kNT + 4) * 4;    // [k-tile (padded)][t][column] uint2
  static constexpr int kCoreTab = (PV ? 512 : 1024) * G;       // CUDA-core q'/p' table
  static constexpr int kTableBytes = kCoreTab > kBTabBytes ? kCoreTab : kBTabBytes;
  static constexpr int kStages0 = (kWarpSmemBudget - kTableBytes - 64) / kStageBytes;
  static constexpr int kStages = kStages0 > 4 ? 4 : (kStages0 < 1 ? 1 : kStages0);
  static constexpr int kWarpSmem = ((kStages * kStageBytes + kTableBytes + kStages * 16) + 127) / 128 * 128;
  // q' table: channel c = h*kChanPerChunk + cc stored at ((cc/4)*NH + h)*4 + cc%4
  static constexpr int kNH = 128 / kChanPerChunk;
};

// q' table of q·Kᵀ: (q'_c, q'_c) pairs; channel c = h*kChanPerChunk + cc sits at float2
// index ((cc/2)*NH + h)*2 + cc%2, so one 16-byte load gives a lane its next two channels.
template <int BITS, int G, bool PV>
__device__ __forceinline__ int table_index(int c) {
  using C = Cfg<BITS, G, PV>;
  const int h = c / C::kChanPerChunk, cc = c % C::kChanPerChunk;
  return ((cc >> 1) * C::kNH + h) * 2 + (cc & 1);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Warp-private shared memory region.
template <int BITS, int G, bool PV>
struct WarpMem {
  using C = Cfg<BITS, G, PV>;
  unsigned char* base;
  __device__ unsigned char* stage(int s) const { return base + s * C::kStageBytes; }
  __device__ float* table() const { return reinterpret_cast<float*>(base + C::kStages * C::kStageBytes); }
  __device__ uint64_t* bar(int s) const {
    return reinterpret_cast<uint64_t*>(base + C::kStages * C::kStageBytes + C::kTableBytes) + s;
  }
  __device__ int* kind(int s) const {
    return reinterpret_cast<int*>(base + C::kStages * C::kStageBytes + C::kTableBytes + C::kStages * 8) + s;
  }
};

// Position in the flat item list: (sequence*kv_heads + head, item within it).
struct Cursor {
  long bh;
  int j;
  __device__ void next(int items_per_bh) {
    if (++j == items_per_bh) {
      j = 0;
      ++bh;
    }
  }
};

// Index entry {offset16, length16} of item c ({0, 0} for a tail item).  Loaded one
// item ahead of its use so that its latency hides behind a block's arithmetic.
__device__ __forceinline__ uint2 index_entry(const GemvArgs& a, Cursor c) {
  if (c.j >= a.n_blocks) return make_uint2(0u, 0u);
  return *reinterpret_cast<const uint2*>(a.index + ((size_t)c.bh * a.max_blocks + c.j) * 2);
}

// Issue the copies of item (bh, j) with index entry e into stage s (whole warp participates).
template <int BITS, int G, bool PV>
__device__ __forceinline__ void issue_item(const GemvArgs& a, const WarpMem<BITS, G, PV>& m, Cursor c, uint2 e,
                                           int s, int lane) {
  using C = Cfg<BITS, G, PV>;
  const long bh = c.bh;
  const int j = c.j;
  int kind = kKindTail;
  uint64_t off16 = 0;
  uint32_t len16 = 0;
  if (j < a.n_blocks) {
    off16 = e.x;
    len16 = e.y;
    const bool valid = e.x != 0xFFFFFFFFu && len16 >= 1040 / 16 && len16 * 16u <= (uint32_t)C::kRecBytes &&
                       off16 + len16 <= a.arena16;
    kind = !valid ? kKindInvalid : (len16 * 16u == (uint32_t)C::kRecBytes ? kKindRaw : kKindPacked);
  }
  unsigned char* st = m.stage(s);
  const unsigned char* src = a.arena + off16 * 16;
  if (lane == 0) {
    *m.kind(s) = kind;
    uint32_t bytes = 0;
    if (kind == kKindRaw) bytes = C::kRecBytes;
    if (kind == kKindPacked) bytes = len16 * 16u;
    if (PV && bytes) bytes += 512u * G;
    fence_async_smem();
    if (bytes)
      mbar_arrive_expect_tx(m.bar(s), bytes);
    else
      mbar_arrive(m.bar(s));
  }
  __syncwarp();
  if (kind == kKindRaw && C::kChunked) {
    if (lane < C::kChunks)
      bulk_g2s(st + 528 + lane * C::kPitch, src + 528 + lane * C::kChunkBytes, C::kChunkBytes, m.bar(s));
    if (lane == 16) bulk_g2s(st, src, 528, m.bar(s));
  } else if (kind == kKindRaw) {
    if (lane == 16) bulk_g2s(st, src, C::kRecBytes, m.bar(s));
  } else if (kind == kKindPacked) {
    if (lane == 16) bulk_g2s(st, src, len16 * 16u, m.bar(s));
  }
  if (PV && (kind == kKindRaw || kind == kKindPacked) && lane >= 24 && lane < 24 + G) {
    const int hd = lane - 24;
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    const long hq = h * G + hd;
    const float* prow = a.p + ((size_t)b * a.kv_heads * G + hq) * a.ld + (size_t)j * 128;
    bulk_g2s(st + C::kStageRec + hd * 512, prow, 512, m.bar(s));
  }
}

// ----------------------------------------------------------------------------
// Tensor-core decode of raw b = 2 / 4 records (fragment order, FORMAT.md section 4)
// ----------------------------------------------------------------------------
// (w & MASK) | 0x64006400: two fields become fp16 1024 + field*2^shift, exactly.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t hfld(uint32_t w) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(0x64006400u));
  return d;
}

// Exact field values from hfld: (1024 + field*2^k) * 2^-k - 1024 * 2^-k = field
// (one fused fp16x2 FMA; every intermediate is an fp16 integer below 2048).
template <uint32_t MASK, int K>
__device__ __forceinline__ uint32_t hval(uint32_t w) {
  const uint32_t bits = hfld<MASK>(w);
  const __half2 x = *reinterpret_cast<const __half2*>(&bits);
  const __half2 mul = __float2half2_rn(1.0f / float(1 << K));
  const __half2 add = __float2half2_rn(-1024.0f / float(1 << K));
  const __half2 r = __hfma2(x, mul, add);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// D += A(16x16, fp16) * B(16x8, fp16), fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Word offset of half kh of the B-table entry (k-tile kt, thread t, column n); the
// k-tile stride is padded by 4 words so that the table's stores spread over banks.
template <int NT>
__device__ __forceinline__ int btab_word(int kt, int t, int n, int kh) {
  return kt * (64 * NT + 4) + (t * 8 * NT + n) * 2 + kh;
}

// Per-block B operand of the MMA: column n = 2*head + part holds, for every k
// (channel for q·Kᵀ, storage slot for p·V), the fp16 high (part 0) or low
// (part 1) half of v[head][k] * f[head]; f is a power of two putting the head's
// largest |v| in [2^14, 2^15).  Summing the two columns of a head restores v to
// about 22 bits.  Table entry [k-tile][t][column] = {b0, b1} of the m16n8k16
// fragment.  Lane holds v for k = 4*lane .. 4*lane+3.  Returns 1/f per head.
template <int G, int NT>
__device__ __forceinline__ void build_btab(uint32_t* btab, const float (&v)[G][4], float (&invf)[G], int lane) {
  uint32_t pr[G][2][2];  // [head][part][pair]
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    const float mx = warp_max(fmaxf(fmaxf(fabsf(v[hd][0]), fabsf(v[hd][1])), fmaxf(fabsf(v[hd][2]), fabsf(v[hd][3]))));
    const int e = mx > 0.f ? (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127 : 0;
    const float f = mx > 0.f ? exp2i(14 - e) : 1.f;
    invf[hd] = mx > 0.f ? exp2i(e - 14) : 1.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float x0 = v[hd][2 * q] * f, x1 = v[hd][2 * q + 1] * f;
      const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
      const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
      pr[hd][0][q] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
      pr[hd][1][q] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
    }
  }
  // live columns 0 .. 2G-1 only; columns 2G .. 8NT-1 stay zero (zero_btab).  The
  // lane's column order is rotated by its k-tile so that one store instruction
  // spreads over the banks instead of hitting the same bank eight times.
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int k = 4 * lane + 2 * q;  // even: the pair (k, k+1)
    const int kt = k >> 4, kk = k & 15, kh = kk >> 3, t = (kk & 7) >> 1;
    uint32_t* row = btab + btab_word<NT>(kt, t, 0, kh);
#pragma unroll
    for (int i = 0; i < 2 * G; ++i) {
      const int n = (i + kt) % (2 * G);
      uint32_t val = 0u;
#pragma unroll
      for (int c = 0; c < 2 * G; ++c)
        if (n == c) val = pr[c >> 1][c & 1][q];
      row[2 * n] = val;
    }
  }
}

// Zeroes the whole B table (the columns of absent heads must read as zero).
template <int NT>
__device__ __forceinline__ void zero_btab(uint32_t* btab, int lane) {
  uint4* p = reinterpret_cast<uint4*>(btab);
#pragma unroll
  for (int i = lane; i < 8 * (64 * NT + 4) / 4; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
}

// Selects per-thread values of head 4*j + t (the head of MMA columns 2t, 2t+1 in n-tile j).
template <int G>
__device__ __forceinline__ float head_sel(const float (&x)[G], int head) {
  float r = 0.f;
#pragma unroll
  for (int hd = 0; hd < G; ++hd)
    if (head == hd) r = x[hd];
  return r;
}

// One raw b = 2 / 4 K block: scores of all 128 slots for the G heads.
template <int BITS, int G>
__device__ __forceinline__ void qk_tc(const unsigned char* st, const uint32_t* btab, const float (&cst)[G],
                                      const float (&invf)[G], float* srow0, long ld,
                                      float scale, int lane) {
  constexpr int NT = (2 * G + 7) / 8;
  const int g = lane >> 2, t = lane & 3;
  uint32_t bf[NT][8][2];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      const uint2 e = *reinterpret_cast<const uint2*>(btab + btab_word<NT>(kt, t, 8 * j + g, 0));
      bf[j][kt][0] = e.x;
      bf[j][kt][1] = e.y;
    }
  float c_t[NT], f_t[NT];
  bool live[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int head = 4 * j + t;
    live[j] = head < G;
    c_t[j] = head_sel<G>(cst, head);
    f_t[j] = head_sel<G>(invf, head);
  }
  // words (tile pair tp, k-tile kt) of this lane: uint4 index (tp*2 + kt/4)*32 + lane, component kt%4.
  // Each k step issues the MMAs of 4 row tiles: 4 independent accumulator chains.
  const uint4* words = reinterpret_cast<const uint4*>(st + kRawWordOffset);
  constexpr int kWordTiles = BITS == 4 ? 4 : 2;  // word rows per half (b = 2: a word feeds two row tiles)
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    uint32_t w[kWordTiles][8];
#pragma unroll
    for (int u = 0; u < kWordTiles; ++u) {
      const int tp = half * kWordTiles + u;
      const uint4 wa = words[(tp * 2) * 32 + lane], wb = words[(tp * 2 + 1) * 32 + lane];
      w[u][0] = wa.x; w[u][1] = wa.y; w[u][2] = wa.z; w[u][3] = wa.w;
      w[u][4] = wb.x; w[u][5] = wb.y; w[u][6] = wb.z; w[u][7] = wb.w;
    }
    float d[4][NT][4];  // 4 row tiles
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[u][j][i] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
#pragma unroll
      for (int u = 0; u < kWordTiles; ++u) {
        const uint32_t x = w[u][kt], h = x >> 8;
        if constexpr (BITS == 4) {
          const uint32_t r0 = hval<0x000F000Fu, 0>(x), r1 = hval<0x00F000F0u, 4>(x);
          const uint32_t r2 = hval<0x000F000Fu, 0>(h), r3 = hval<0x00F000F0u, 4>(h);
#pragma unroll
          for (int j = 0; j < NT; ++j) mma16816(d[u][j], r0, r1, r2, r3, bf[j][kt][0], bf[j][kt][1]);
        } else {
          const uint32_t r0 = hval<0x00030003u, 0>(x), r1 = hval<0x000C000Cu, 2>(x);
          const uint32_t r2 = hval<0x00030003u, 0>(h), r3 = hval<0x000C000Cu, 2>(h);
          const uint32_t s0 = hval<0x00300030u, 4>(x), s1 = hval<0x00C000C0u, 6>(x);
          const uint32_t s2 = hval<0x00300030u, 4>(h), s3 = hval<0x00C000C0u, 6>(h);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            mma16816(d[2 * u][j], r0, r1, r2, r3, bf[j][kt][0], bf[j][kt][1]);
            mma16816(d[2 * u + 1][j], s0, s1, s2, s3, bf[j][kt][0], bf[j][kt][1]);
          }
        }
      }
    }
    // row tile u of this half covers slots 16*(4*half + u) + g and + 8
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (!live[j]) continue;
      float* dst = srow0 + (4 * j + t) * ld;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 16 * (4 * half + u) + g;
        dst[r] = scale * fmaf(d[u][j][0] + d[u][j][1], f_t[j], c_t[j]);
        dst[r + 8] = scale * fmaf(d[u][j][2] + d[u][j][3], f_t[j], c_t[j]);
      }
    }
  }
}

// One raw b = 2 / 4 V block: adds sum_slots p'*v_hat into the per-thread fp32
// accumulators of channels 16*T + g (acc_lo) and 16*T + g + 8 (acc_hi), head 4j + t.
template <int BITS, int G>
__device__ __forceinline__ void pv_tc(const unsigned char* st, const uint32_t* btab,
                                      const float (&invf)[G], float (&acc_lo)[(2 * G + 7) / 8][8],
                                      float (&acc_hi)[(2 * G + 7) / 8][8], int lane) {
  constexpr int NT = (2 * G + 7) / 8;
  const int g = lane >> 2, t = lane & 3;
  uint32_t bf[NT][8][2];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      const uint2 e = *reinterpret_cast<const uint2*>(btab + btab_word<NT>(kt, t, 8 * j + g, 0));
      bf[j][kt][0] = e.x;
      bf[j][kt][1] = e.y;
    }
  float f_t[NT];
  bool live[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    live[j] = 4 * j + t < G;
    f_t[j] = head_sel<G>(invf, 4 * j + t);
  }
  const uint4* words = reinterpret_cast<const uint4*>(st + kRawWordOffset);
  constexpr int kWordTiles = BITS == 4 ? 4 : 2;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t w[kWordTiles][8];
#pragma unroll
    for (int u = 0; u < kWordTiles; ++u) {
      const int tp = half * kWordTiles + u;
      const uint4 wa = words[(tp * 2) * 32 + lane], wb = words[(tp * 2 + 1) * 32 + lane];
      w[u][0] = wa.x; w[u][1] = wa.y; w[u][2] = wa.z; w[u][3] = wa.w;
      w[u][4] = wb.x; w[u][5] = wb.y; w[u][6] = wb.z; w[u][7] = wb.w;
    }
    float d[4][NT][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[u][j][i] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
#pragma unroll
      for (int u = 0; u < kWordTiles; ++u) {
        const uint32_t x = w[u][kt], h = x >> 8;
        if constexpr (BITS == 4) {
          const uint32_t r0 = hval<0x000F000Fu, 0>(x), r1 = hval<0x00F000F0u, 4>(x);
          const uint32_t r2 = hval<0x000F000Fu, 0>(h), r3 = hval<0x00F000F0u, 4>(h);
#pragma unroll
          for (int j = 0; j < NT; ++j) mma16816(d[u][j], r0, r1, r2, r3, bf[j][kt][0], bf[j][kt][1]);
        } else {
          const uint32_t r0 = hval<0x00030003u, 0>(x), r1 = hval<0x000C000Cu, 2>(x);
          const uint32_t r2 = hval<0x00030003u, 0>(h), r3 = hval<0x000C000Cu, 2>(h);
          const uint32_t s0 = hval<0x00300030u, 4>(x), s1 = hval<0x00C000C0u, 6>(x);
          const uint32_t s2 = hval<0x00300030u, 4>(h), s3 = hval<0x00C000C0u, 6>(h);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            mma16816(d[2 * u][j], r0, r1, r2, r3, bf[j][kt][0], bf[j][kt][1]);
            mma16816(d[2 * u + 1][j], s0, s1, s2, s3, bf[j][kt][0], bf[j][kt][1]);
          }
        }
      }
    }
    // row tile u of this half covers channels 16*(4*half + u) + g and + 8
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (!live[j]) continue;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc_lo[j][4 * half + u] = fmaf(d[u][j][0] + d[u][j][1], f_t[j], acc_lo[j][4 * half + u]);
        acc_hi[j][4 * half + u] = fmaf(d[u][j][2] + d[u][j][3], f_t[j], acc_hi[j][4 * half + u]);
      }
    }
  }
}

// ----------------------------------------------------------------------------
// q·Kᵀ
// ----------------------------------------------------------------------------
template <int BITS, int G>
__device__ __forceinline__ void qk_raw(const unsigned char* st, const float2* qp, const float (&cst)[G],
                                       float* srow0, long ld, float scale, int lane) {
  using C = Cfg<BITS, G, false>;
  if constexpr (BITS == 4) {
    // lane = (group g, token octet k, channel half h); word k of unit (g, c) holds tokens 32g+8k..+7
    const int h = lane & 1, k = (lane >> 1) & 3, g = lane >> 3;
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (2 * g + h) * C::kPitch) + k;
    float2 acc[G][4];
#pragma unroll
    for (int hd = 0; hd < G; ++hd)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[hd][i] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int c2 = 0; c2 < 32; ++c2) {
      float2 v0[4], v1[4];
      dec4(wp[8 * c2], v0);
      dec4(wp[8 * c2 + 4], v1);
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 qq = *reinterpret_cast<const float4*>(qp + hd * 128 + (c2 * C::kNH + h) * 2);
        const float2 q0 = make_float2(qq.x, qq.y), q1 = make_float2(qq.z, qq.w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[hd][i] = __ffma2_rn(q0, v0[i], acc[hd][i]);
          acc[hd][i] = __ffma2_rn(q1, v1[i], acc[hd][i]);
        }
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      float t[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        t[2 * i] = acc[hd][i].x + __shfl_xor_sync(0xffffffffu, acc[hd][i].x, 1);
        t[2 * i + 1] = acc[hd][i].y + __shfl_xor_sync(0xffffffffu, acc[hd][i].y, 1);
      }
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = t[i] * pow2(-sig4(i));
        const float hi = t[i + 4] * pow2(-sig4(i + 4));
        o[i] = scale * (cst[hd] + (h ? hi : lo));
      }
      float* dst = srow0 + hd * ld + 32 * g + 8 * k + 4 * h;
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    }
  } else {
    // lane = (group g, 16-token half k, channel quarter h)
    const int h = lane & 3, k = (lane >> 2) & 1, g = lane >> 3;
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (4 * g + h) * C::kPitch);
    float2 acc[G][8];
#pragma unroll
    for (int hd = 0; hd < G; ++hd)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[hd][i] = make_float2(0.f, 0.f);
#pragma unroll 2
    for (int c2 = 0; c2 < 16; ++c2) {
      float2 v0[8], v1[8];
      if constexpr (BITS == 2) {
        dec2(wp[2 * (2 * c2) + k], v0);
        dec2(wp[2 * (2 * c2 + 1) + k], v1);
      } else {
        dec3(wp[3 * (2 * c2) + k], wp[3 * (2 * c2) + 2] >> (16 * k), v0);
        dec3(wp[3 * (2 * c2 + 1) + k], wp[3 * (2 * c2 + 1) + 2] >> (16 * k), v1);
      }
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 qq = *reinterpret_cast<const float4*>(qp + hd * 128 + (c2 * C::kNH + h) * 2);
        const float2 q0 = make_float2(qq.x, qq.y), q1 = make_float2(qq.z, qq.w);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc[hd][i] = __ffma2_rn(q0, v0[i], acc[hd][i]);
          acc[hd][i] = __ffma2_rn(q1, v1[i], acc[hd][i]);
        }
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      float t[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float x = acc[hd][i].x, y = acc[hd][i].y;
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        y += __shfl_xor_sync(0xffffffffu, y, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        y += __shfl_xor_sync(0xffffffffu, y, 2);
        t[2 * i] = x;
        t[2 * i + 1] = y;
      }
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = 0.f;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh)
          if (h == hh) v = t[4 * hh + i] * pow2(-sig2(4 * hh + i));
        o[i] = scale * (cst[hd] + v);
      }
      float* dst = srow0 + hd * ld + 32 * g + 16 * k + 4 * h;
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Extracts the offset of token j from a compressed unit of width w starting at word s.
__device__ __forceinline__ uint32_t unit_field(const uint32_t* W, int s, int w, int j) {
  uint32_t u = 0;
  if (w == 4) {
    u = (W[s + (j >> 3)] >> ((j & 7) * 4)) & 15u;
  } else if (w >= 2) {
    u = (W[s + (j >> 4)] >> ((j & 15) * 2)) & 3u;
    if (w == 3) u |= ((W[s + 2] >> j) & 1u) << 2;
  } else if (w == 1) {
    u = (W[s] >> j) & 1u;
  }
  return u;
}

template <int BITS, int G>
__device__ __forceinline__ void qk_packed(const unsigned char* st, const float2* qp, const float (&cst)[G],
                                          float* srow0, long ld, float scale, int lane) {
  const uint16_t* gws = reinterpret_cast<const uint16_t*>(st);
  const uint8_t* meta = st + kMetaOffset;
  const uint32_t* W = reinterpret_cast<const uint32_t*>(st + kPackedWordOffset);
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    // base term of this group: sum_c q'_c base_gc, lane covers channels 4*lane..4*lane+3
    float bsum[G];
    const uint32_t m4 = *reinterpret_cast<const uint32_t*>(meta + g * 128 + 4 * lane);
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        part = fmaf(qp[hd * 128 + table_index<BITS, G, false>(4 * lane + i)].x, (float)((m4 >> (8 * i)) & 15u), part);
      bsum[hd] = warp_sum(part);
    }
    float acc[G];
#pragma unroll
    for (int hd = 0; hd < G; ++hd) acc[hd] = 0.f;
    int s = gws[g];
#pragma unroll 1
    for (int c4 = 0; c4 < 32; ++c4) {
      const uint32_t mm = *reinterpret_cast<const uint32_t*>(meta + g * 128 + 4 * c4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = (mm >> (8 * i + 4)) & 15u;
        const float u = (float)unit_field(W, s, w, lane);
        s += w;
#pragma unroll
        for (int hd = 0; hd < G; ++hd)
          acc[hd] = fmaf(qp[hd * 128 + table_index<BITS, G, false>(4 * c4 + i)].x, u, acc[hd]);
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) srow0[hd * ld + 32 * g + lane] = scale * (cst[hd] + bsum[hd] + acc[hd]);
  }
}

template <int G>
__device__ __forceinline__ void qk_tail(const GemvArgs& a, long bh, const float (&qr)[G][4], float* srow0,
                                        int lane) {
  const uint16_t* tail = a.tail + (size_t)bh * 128 * 128;
  for (int t0 = 0; t0 < a.tail_len; t0 += 32) {
    float mine[G];
#pragma unroll
    for (int hd = 0; hd < G; ++hd) mine[hd] = 0.f;
    const int tn = min(32, a.tail_len - t0);
    for (int t = 0; t < tn; ++t) {
      const uint2 hv = *reinterpret_cast<const uint2*>(tail + (size_t)(t0 + t) * 128 + 4 * lane);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        float part = qr[hd][0] * f0.x;
        part = fmaf(qr[hd][1], f0.y, part);
        part = fmaf(qr[hd][2], f1.x, part);
        part = fmaf(qr[hd][3], f1.y, part);
        part = warp_sum(part);
        if (lane == t) mine[hd] = part;
      }
    }
    if (lane < tn) {
#pragma unroll
      for (int hd = 0; hd < G; ++hd) srow0[hd * a.ld + (long)a.n_blocks * 128 + t0 + lane] = a.scale * mine[hd];
    }
  }
}

template <int BITS, int G>
__global__ void __launch_bounds__(kWarpsPerCta * 32) qk_kernel(const GemvArgs a) {
  using C = Cfg<BITS, G, false>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (warp >= a.n_warps) return;
  WarpMem<BITS, G, false> m{smem + (threadIdx.x >> 5) * C::kWarpSmem};
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(m.bar(s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  long prod = lo;
  Cursor pc{lo / a.items_per_bh, (int)(lo % a.items_per_bh)};
  Cursor cc = pc;
  for (int s = 0; s < C::kStages && prod < hi; ++s, ++prod, pc.next(a.items_per_bh))
    issue_item<BITS, G, false>(a, m, pc, index_entry(a, pc), s, lane);
  uint2 next_e = prod < hi ? index_entry(a, pc) : make_uint2(0u, 0u);

  const int q_heads = a.kv_heads * G;
  long cur_bh = -1;
  bool btab_clean = false;  // the table region holds a B table whose absent-head columns are zero
  float qr[G][4];
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x, cc.next(a.items_per_bh)) {
    const long bh = cc.bh;
    const int j = cc.j;
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    float* srow0 = a.scores + ((size_t)b * q_heads + h * G) * a.ld;
    if (bh != cur_bh) {
      cur_bh = bh;
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const uint2 hv = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * q_heads + h * G + hd) * 128 + 4 * lane);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
        qr[hd][0] = f0.x;
        qr[hd][1] = f0.y;
        qr[hd][2] = f1.x;
        qr[hd][3] = f1.y;
      }
    }
    const bool ok = mbar_wait_bounded(m.bar(s), (phases >> s) & 1u, a.ctrl);
    phases ^= 1u << s;
    if (!ok) return;  // the copy never landed: stop this warp (status already set)
    const int kind = *m.kind(s);
    const unsigned char* st = m.stage(s);
    if (kind == kKindTail) {
      qk_tail<G>(a, bh, qr, srow0, lane);
    } else if (kind == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
#pragma unroll
      for (int hd = 0; hd < G; ++hd)
        for (int i = lane; i < 128; i += 32) srow0[hd * a.ld + (long)j * 128 + i] = __int_as_float(0x7fc00000);
    } else {
      // per block: the min term sum_c q_c * mn_c, then q' = q * scale_c as the
      // tensor-core B table (raw b = 2 / 4) or the CUDA-core q' table
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      float cst[G];
      float qv[G][4];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        float part = qr[hd][0] * mn0.x;
        part = fmaf(qr[hd][1], mn0.y, part);
        part = fmaf(qr[hd][2], mn1.x, part);
        part = fmaf(qr[hd][3], mn1.y, part);
        cst[hd] = warp_sum(part);
        qv[hd][0] = qr[hd][0] * sc0.x;
        qv[hd][1] = qr[hd][1] * sc0.y;
        qv[hd][2] = qr[hd][2] * sc1.x;
        qv[hd][3] = qr[hd][3] * sc1.y;
      }
      float* sblk = srow0 + (long)j * 128;
      if (kind == kKindRaw && !C::kChunked) {
        uint32_t* btab = reinterpret_cast<uint32_t*>(m.table());
        if (!btab_clean) zero_btab<C::kNT>(btab, lane);
        btab_clean = true;
        float invf[G];
        build_btab<G, C::kNT>(btab, qv, invf, lane);
        __syncwarp();
        qk_tc<BITS, G>(st, btab, cst, invf, sblk, a.ld, a.scale, lane);
      } else {
        btab_clean = false;
        float2* qp = reinterpret_cast<float2*>(m.table());
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          *reinterpret_cast<float4*>(qp + hd * 128 + table_index<BITS, G, false>(4 * lane)) =
              make_float4(qv[hd][0], qv[hd][0], qv[hd][1], qv[hd][1]);
          *reinterpret_cast<float4*>(qp + hd * 128 + table_index<BITS, G, false>(4 * lane + 2)) =
              make_float4(qv[hd][2], qv[hd][2], qv[hd][3], qv[hd][3]);
        }
        __syncwarp();
        if (kind == kKindRaw)
          qk_raw<BITS, G>(st, qp, cst, sblk, a.ld, a.scale, lane);
        else
          qk_packed<BITS, G>(st, qp, cst, sblk, a.ld, a.scale, lane);
      }
    }
    __syncwarp();
    if (prod < hi) {
      issue_item<BITS, G, false>(a, m, pc, next_e, s, lane);
      ++prod;
      pc.next(a.items_per_bh);
      if (prod < hi) next_e = index_entry(a, pc);
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
}

// ----------------------------------------------------------------------------
// p·V
// ----------------------------------------------------------------------------
// Accumulates one raw block into acc[slab][hd] (lane = channel slab*32 + lane).  The
// field exponents are folded into p'' = p * scale * 2^-sig, so decoded pairs multiply
// consecutive p'' pairs directly.
template <int BITS, int G>
__device__ __forceinline__ void pv_raw(const unsigned char* st, const float* pp, float2 (&acc)[4][G], int lane) {
  using C = Cfg<BITS, G, true>;
  constexpr bool kRegP = G <= 2;  // keep the group's p'' in registers across the 4 slabs
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    float2 pr[kRegP ? G : 1][16];
    if constexpr (kRegP) {
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4* p4 = reinterpret_cast<const float4*>(pp + hd * 128 + 32 * g);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 x = p4[q];
          pr[hd][2 * q] = make_float2(x.x, x.y);
          pr[hd][2 * q + 1] = make_float2(x.z, x.w);
        }
      }
    }
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      float2 v[16];
      if constexpr (BITS == 4) {
        const uint4 u = *reinterpret_cast<const uint4*>(st + 528 + (2 * g + (sl >> 1)) * C::kPitch +
                                                        ((sl & 1) * 32 + lane) * 16);
        float2 t[4];
        dec4(u.x, t);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = t[i];
        dec4(u.y, t);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[4 + i] = t[i];
        dec4(u.z, t);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[8 + i] = t[i];
        dec4(u.w, t);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[12 + i] = t[i];
      } else if constexpr (BITS == 2) {
        const uint2 u = *reinterpret_cast<const uint2*>(st + 528 + (4 * g + sl) * C::kPitch + lane * 8);
        float2 t[8];
        dec2(u.x, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = t[i];
        dec2(u.y, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 + i] = t[i];
      } else {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (4 * g + sl) * C::kPitch + lane * 12);
        const uint32_t w0 = wp[0], w1 = wp[1], w2 = wp[2];
        float2 t[8];
        dec3(w0, w2, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = t[i];
        dec3(w1, w2 >> 16, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 + i] = t[i];
      }
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        float2 a0 = acc[sl][hd], a1 = make_float2(0.f, 0.f);
        if constexpr (kRegP) {
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            a0 = __ffma2_rn(pr[hd][i], v[i], a0);
            a1 = __ffma2_rn(pr[hd][i + 1], v[i + 1], a1);
          }
        } else {
          const float4* p4 = reinterpret_cast<const float4*>(pp + hd * 128 + 32 * g);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 x = p4[q];
            a0 = __ffma2_rn(make_float2(x.x, x.y), v[2 * q], a0);
            a1 = __ffma2_rn(make_float2(x.z, x.w), v[2 * q + 1], a1);
          }
        }
        acc[sl][hd] = __fadd2_rn(a0, a1);
      }
    }
  }
}

template <int BITS, int G>
__device__ __forceinline__ void pv_packed(const unsigned char* st, const float* pp, const float (&pg)[G][4],
                                          float2 (&acc)[4][G], int lane) {
  const uint16_t* gws = reinterpret_cast<const uint16_t*>(st);
  const uint8_t* meta = st + kMetaOffset;
  const uint32_t* W = reinterpret_cast<const uint32_t*>(st + kPackedWordOffset);
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    int carry = gws[g];
#pragma unroll 1
    for (int sl = 0; sl < 4; ++sl) {
      const int c = sl * 32 + lane;
      const uint32_t mb = meta[g * 128 + c];
      const int w = (int)(mb >> 4), base = (int)(mb & 15u);
      int incl = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int start = carry + incl - w;
      carry += __shfl_sync(0xffffffffu, incl, 31);
#pragma unroll 1
      for (int hd = 0; hd < G; ++hd) {
        const float* pr = pp + hd * 128 + 32 * g;
        float sum = (float)base * pg[hd][g];
        if (w == 4) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t word = W[start + q];
#pragma unroll
            for (int i = 0; i < 8; ++i) sum = fmaf(pr[8 * q + i], (float)((word >> (4 * i)) & 15u), sum);
          }
        } else {
          int at = start;
          float lo_mul = 1.f;
          if (w & 2) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t word = W[at + q];
#pragma unroll
              for (int i = 0; i < 16; ++i) sum = fmaf(pr[16 * q + i], (float)((word >> (2 * i)) & 3u), sum);
            }
            at += 2;
            lo_mul = 4.f;
          }
          if (w & 1) {
            const uint32_t word = W[at];
            float s1 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) s1 = fmaf(pr[i], (float)((word >> i) & 1u), s1);
            sum = fmaf(lo_mul, s1, sum);
          }
        }
        acc[sl][hd].x += sum;
      }
    }
  }
}

// Writes this warp's partial sums for (b, h) to its slot (warp + bh) and clears
// them.  The tensor-core accumulators (thread (g, t) holds channels 16T+g and
// 16T+g+8 of head 4j+t) go through `buf` (G x 128 floats of warp shared memory)
// to the lane = channel layout of the CUDA-core accumulators.
template <int G>
__device__ __forceinline__ void pv_flush(const GemvArgs& a, long bh, int warp, float2 (&acc)[4][G],
                                         float (&acc_lo)[(2 * G + 7) / 8][8], float (&acc_hi)[(2 * G + 7) / 8][8],
                                         float (&mp)[G], float* buf, int lane) {
  constexpr int NT = (2 * G + 7) / 8;
  const int g = lane >> 2, t = lane & 3;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int head = 4 * j + t;
#pragma unroll
    for (int T = 0; T < 8; ++T) {
      if (head < G) {
        buf[head * 128 + 16 * T + g] = acc_lo[j][T];
        buf[head * 128 + 16 * T + g + 8] = acc_hi[j][T];
      }
      acc_lo[j][T] = 0.f;
      acc_hi[j][T] = 0.f;
    }
  }
  __syncwarp();
  float* part = a.partials + (size_t)(warp + bh) * G * 128;
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    const float mn = warp_sum(mp[hd]);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int c = sl * 32 + lane;
      __stcg(part + hd * 128 + c, buf[hd * 128 + c] + acc[sl][hd].x + acc[sl][hd].y + mn);
      acc[sl][hd] = make_float2(0.f, 0.f);
    }
    mp[hd] = 0.f;
  }
  __syncwarp();
}

// Warp whose item range holds `item` (ranges are [floor(w*N/W), floor((w+1)*N/W)), W <= N).
__device__ __forceinline__ long warp_of_item(long item, long n_items, long n_warps) {
  return (long)(((long long)(item + 1) * n_warps + n_items - 1) / n_items) - 1;
}

// Second pass of p·V: out = sum of the partials of every warp that touched
// (b, h), in a fixed order (deterministic).  One CTA per output row (b, h, head):
// warp i of 8 adds partial slots w0+i, w0+i+8, ... with coalesced 16-byte loads,
// then warp 0 adds the 8 warp sums in order.  It is launched as a programmatic
// dependent of pv_kernel and waits for its results.
template <int G>
__global__ void __launch_bounds__(256) pv_reduce_kernel(const GemvArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float4 warp_sum4[8][32];
  const long row = blockIdx.x;  // (b*kv_heads + h)*G + head
  const long bh = row / G;
  const int hd = (int)(row % G);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long I = a.items_per_bh;
  const long w0 = warp_of_item(bh * I, a.n_items, a.n_warps);
  const long w1 = warp_of_item((bh + 1) * I - 1, a.n_items, a.n_warps);
  const float4* base = reinterpret_cast<const float4*>(a.partials + ((size_t)bh * G + hd) * 128) + lane;
  const size_t slot_stride = (size_t)G * 128 / 4;  // float4 per partial slot
  float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
  long w = w0 + warp;
  for (; w + 8 <= w1; w += 16) {
    const float4 x = __ldcg(base + (size_t)w * slot_stride);
    const float4 y = __ldcg(base + (size_t)(w + 8) * slot_stride);
    s0.x += x.x; s0.y += x.y; s0.z += x.z; s0.w += x.w;
    s1.x += y.x; s1.y += y.y; s1.z += y.z; s1.w += y.w;
  }
  if (w <= w1) {
    const float4 x = __ldcg(base + (size_t)w * slot_stride);
    s0.x += x.x; s0.y += x.y; s0.z += x.z; s0.w += x.w;
  }
  warp_sum4[warp][lane] = make_float4(s0.x + s1.x, s0.y + s1.y, s0.z + s1.z, s0.w + s1.w);
  __syncthreads();
  if (warp == 0) {
    float4 r = warp_sum4[0][lane];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      const float4 x = warp_sum4[i][lane];
      r.x += x.x; r.y += x.y; r.z += x.z; r.w += x.w;
    }
    reinterpret_cast<float4*>(a.out + row * 128)[lane] = r;
  }
}

template <int BITS, int G>
__global__ void __launch_bounds__(kWarpsPerCta * 32) pv_kernel(const GemvArgs a) {
  using C = Cfg<BITS, G, true>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (warp >= a.n_warps) return;
  WarpMem<BITS, G, true> m{smem + (threadIdx.x >> 5) * C::kWarpSmem};
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(m.bar(s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  long prod = lo;
  Cursor pc{lo / a.items_per_bh, (int)(lo % a.items_per_bh)};
  Cursor cc = pc;
  for (int s = 0; s < C::kStages && prod < hi; ++s, ++prod, pc.next(a.items_per_bh))
    issue_item<BITS, G, true>(a, m, pc, index_entry(a, pc), s, lane);
  uint2 next_e = prod < hi ? index_entry(a, pc) : make_uint2(0u, 0u);

  float2 acc[4][G];  // CUDA-core paths: lane = channel sl*32 + lane
  float mp[G];
  float acc_lo[C::kNT][8], acc_hi[C::kNT][8];  // tensor-core path
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    mp[hd] = 0.f;
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int jn = 0; jn < C::kNT; ++jn)
#pragma unroll
    for (int T = 0; T < 8; ++T) acc_lo[jn][T] = acc_hi[jn][T] = 0.f;
  float* buf = m.table();
  bool btab_clean = false;  // the table region holds a B table whose absent-head columns are zero
  long cur_bh = cc.bh;
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x, cc.next(a.items_per_bh)) {
    const long bh = cc.bh;
    const int j = cc.j;
    if (bh != cur_bh) {
      pv_flush<G>(a, cur_bh, warp, acc, acc_lo, acc_hi, mp, buf, lane);
      btab_clean = false;  // the flush used the table region as its buffer
      cur_bh = bh;
    }
    const bool ok = mbar_wait_bounded(m.bar(s), (phases >> s) & 1u, a.ctrl);
    phases ^= 1u << s;
    if (!ok) return;
    const int kind = *m.kind(s);
    const unsigned char* st = m.stage(s);
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    if (kind == kKindTail) {
      const uint16_t* tail = a.tail + (size_t)bh * 128 * 128;
      for (int t = 0; t < a.tail_len; ++t) {
        float vv[4];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) vv[sl] = half_bits_to_float(tail[(size_t)t * 128 + sl * 32 + lane]);
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          const float pt = a.p[((size_t)b * a.kv_heads * G + h * G + hd) * a.ld + (long)a.n_blocks * 128 + t];
#pragma unroll
          for (int sl = 0; sl < 4; ++sl) acc[sl][hd].x = fmaf(pt, vv[sl], acc[sl][hd].x);
        }
      }
    } else if (kind == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
    } else {
      // p' = p * scale_r per storage slot and the min term sum_r p_r * mn_r
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      const float mnr[4] = {mn0.x, mn0.y, mn1.x, mn1.y};
      const float scr[4] = {sc0.x, sc0.y, sc1.x, sc1.y};
      float pv4[G][4];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 p4 = *reinterpret_cast<const float4*>(st + C::kStageRec + hd * 512 + 16 * lane);
        const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mp[hd] = fmaf(pr[i], mnr[i], mp[hd]);
          pv4[hd][i] = pr[i] * scr[i];
        }
      }
      if (kind == kKindRaw && !C::kChunked) {
        uint32_t* btab = reinterpret_cast<uint32_t*>(m.table());
        if (!btab_clean) zero_btab<C::kNT>(btab, lane);
        btab_clean = true;
        float invf[G];
        build_btab<G, C::kNT>(btab, pv4, invf, lane);
        __syncwarp();
        pv_tc<BITS, G>(st, btab, invf, acc_lo, acc_hi, lane);
      } else {
        btab_clean = false;
        float* pp = m.table();
        float pg[G][4];
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          float o[4];
          float ps = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            ps += pv4[hd][i];
            const int r15 = (4 * lane + i) & 15;  // field position of slot r in a 2-bit slice word
            const int sg = r15 <= 10 ? 2 * r15 : 2 * r15 - 12;
            o[i] = kind == kKindRaw ? pv4[hd][i] * exp2i(-sg) : pv4[hd][i];  // exact power-of-two scaling
          }
          *reinterpret_cast<float4*>(pp + hd * 128 + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
          if (kind != kKindRaw) {
            // per-group sum of p' (lanes 8g..8g+7 hold group g)
            ps += __shfl_xor_sync(0xffffffffu, ps, 1);
            ps += __shfl_xor_sync(0xffffffffu, ps, 2);
            ps += __shfl_xor_sync(0xffffffffu, ps, 4);
#pragma unroll
            for (int g = 0; g < 4; ++g) pg[hd][g] = __shfl_sync(0xffffffffu, ps, 8 * g);
          }
        }
        __syncwarp();
        if (kind == kKindRaw)
          pv_raw<BITS, G>(st, pp, acc, lane);
        else
          pv_packed<BITS, G>(st, pp, pg, acc, lane);
      }
    }
    __syncwarp();
    if (prod < hi) {
      issue_item<BITS, G, true>(a, m, pc, next_e, s, lane);
      ++prod;
      pc.next(a.items_per_bh);
      if (prod < hi) next_e = index_entry(a, pc);
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
  pv_flush<G>(a, cur_bh, warp, acc, acc_lo, acc_hi, mp, buf, lane);
}

// ----------------------------------------------------------------------------
// Host side: instantiation table, occupancy, launch
// ----------------------------------------------------------------------------
struct KernelInfo {
  const void* fn;
  int smem;
};

template <int BITS, int G, bool PV>
KernelInfo kernel_info() {
  using C = Cfg<BITS, G, PV>;
  if constexpr (PV)
    return {reinterpret_cast<const void*>(&pv_kernel<BITS, G>), kWarpsPerCta * C::kWarpSmem};
  else
    return {reinterpret_cast<const void*>(&qk_kernel<BITS, G>), kWarpsPerCta * C::kWarpSmem};
}

template <bool PV>
bool select(int bits, int group, KernelInfo* out) {
#define PACKKV_CASE(B, GG)                  \
  if (bits == B && group == GG) {           \
    *out = kernel_info<B, GG, PV>();        \
    return true;                            \
  }
  PACKKV_CASE(4, 1) PACKKV_CASE(4, 2) PACKKV_CASE(4, 4) PACKKV_CASE(4, 8)
  PACKKV_CASE(3, 1) PACKKV_CASE(3, 2) PACKKV_CASE(3, 4) PACKKV_CASE(3, 8)
  PACKKV_CASE(2, 1) PACKKV_CASE(2, 2) PACKKV_CASE(2, 4) PACKKV_CASE(2, 8)
#undef PACKKV_CASE
  return false;
}

struct DevKernelKey {
  int dev;
  const void* fn;
  bool operator==(const DevKernelKey& o) const { return dev == o.dev && fn == o.fn; }
};
struct DevKernelHash {
  size_t operator()(const DevKernelKey& k) const { return std::hash<const void*>()(k.fn) ^ (size_t)k.dev; }
};

// Resident warps of `info` on the current device (configures the smem limit once).
cudaError_t resident_warps(const KernelInfo& info, int* warps) {
  static std::mutex mu;
  static std::unordered_map<DevKernelKey, int, DevKernelHash> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, info.fn});
  if (it != cache.end()) {
    *warps = it->second;
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(info.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, info.smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0, sms = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, info.fn, kWarpsPerCta * 32, info.smem);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int w = sms * per_sm * kWarpsPerCta;
  cache[{dev, info.fn}] = w;
  *warps = w;
  return cudaSuccess;
}

template <bool PV>
cudaError_t launch(GemvArgs a, cudaStream_t stream) {
  KernelInfo info{};
  if (!select<PV>(a.bits, a.group, &info)) return cudaErrorInvalidValue;
  int w = 0;
  cudaError_t e = resident_warps(info, &w);
  if (e != cudaSuccess) return e;
  if (w > gemv_max_warps()) w = gemv_max_warps();
  a.n_warps = (int)(a.n_items < w ? a.n_items : w);
  const unsigned grid = (unsigned)((a.n_warps + kWarpsPerCta - 1) / kWarpsPerCta);
  void* args[] = {&a};
  e = cudaLaunchKernel(info.fn, dim3(grid), dim3(kWarpsPerCta * 32), args, info.smem, stream);
  if (e != cudaSuccess || !PV) return e;
  // second pass of p·V, launched early (programmatic dependent launch); it waits for pv_kernel
  const long rows = (long)a.batch * a.kv_heads * a.group;
  const void* red = nullptr;
  switch (a.group) {
    case 1: red = reinterpret_cast<const void*>(&pv_reduce_kernel<1>); break;
    case 2: red = reinterpret_cast<const void*>(&pv_reduce_kernel<2>); break;
    case 4: red = reinterpret_cast<const void*>(&pv_reduce_kernel<4>); break;
    default: red = reinterpret_cast<const void*>(&pv_reduce_kernel<8>); break;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, red, args);
}

}  // namespace

int gemv_max_warps() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * 64;
}

size_t pv_workspace_bytes(int batch, int kv_heads, int group) {
  const size_t bh = (size_t)batch * kv_heads;
  return ((size_t)gemv_max_warps() + bh) * group * 128 * sizeof(float);
}

cudaError_t pv_launch_workspace_bytes(const GemvArgs& a, size_t* bytes) {
  KernelInfo info{};
  if (!select<true>(a.bits, a.group, &info)) return cudaErrorInvalidValue;
  int w = 0;
  const cudaError_t e = resident_warps(info, &w);
  if (e != cudaSuccess) return e;
  if (w > gemv_max_warps()) w = gemv_max_warps();
  const long n_warps = a.n_items < w ? a.n_items : w;
  *bytes = ((size_t)n_warps + (size_t)a.batch * a.kv_heads) * a.group * 128 * sizeof(float);
  return cudaSuccess;
}

cudaError_t launch_qk(GemvArgs a, cudaStream_t stream) { return launch<false>(a, stream); }
cudaError_t launch_pv(GemvArgs a, cudaStream_t stream) { return launch<true>(a, stream); }

}  // namespace packkv
