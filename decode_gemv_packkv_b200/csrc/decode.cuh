// Device building blocks of the fused decode products over the packed cache:
// record staging (bulk copies into warp-private shared-memory stages, bounded
// mbarrier waits), the 8-bit integer tensor-core decode of raw records (2, 3 and
// 4-bit) and of compressed records (q·Kᵀ: units sorted by width; p·V: every slice
// kind decoded and masked by width; packed-cache format v1, sections 3-4).  Included by the q·Kᵀ / p·V kernels and by the fused attention kernel.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace packkv {

namespace {

#ifndef PACKKV_WARPS_PER_CTA
#define PACKKV_WARPS_PER_CTA 4
#endif
constexpr int kWarpsPerCta = PACKKV_WARPS_PER_CTA;
#ifndef PACKKV_WARP_SMEM_KB
#define PACKKV_WARP_SMEM_KB 10  // shared memory per warp: one 4-bit stage, five CTAs of 4 warps per SM
#endif
constexpr int kWarpSmemBudget = PACKKV_WARP_SMEM_KB * 1024;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer in the low bits
constexpr int kRoundBits = 0x4B400000;

enum ItemKind : int { kKindRaw = 0, kKindPacked = 1, kKindInvalid = 2, kKindTail = 3 };

// Columns of the int8 tensor-core B table (q' or p' as three base-128 digits per head)
// and which accumulator values a thread ends with.  A thread (g, t) of an m16n8
// accumulator tile holds columns 2t and 2t + 1.
//  * Paired (G <= 2): n-tile j holds heads 2j, 2j + 1 as columns 4*(head - 2j) + digit
//    (digit 3 zero).  Thread t has digits 0, 1 (even t) or 2 (odd t) of head 2j + t/2;
//    one shuffle joins them into the even-t thread.
//  * Split (G >= 4, a multiple of 4): n-tiles 2i and 2i + 1 hold heads 4i .. 4i + 3:
//    column 2u + d of n-tile 2i is digit d < 2 of head 4i + u, column 2u of n-tile
//    2i + 1 its digit 2 (column 2u + 1 zero).  Thread t has all three digits of head
//    4i + t, so every thread ends with one head's rows and no shuffle is needed.
// kNH accumulator sets per thread, index jh: head(jh, t), owned where owns(jh, t).
#ifndef PACKKV_SPLIT_MIN_G
#define PACKKV_SPLIT_MIN_G 4
#endif
template <int G>
struct I8Layout {
  static constexpr bool kSplit = G >= PACKKV_SPLIT_MIN_G;
  static_assert(!kSplit || G % 4 == 0, "split layout takes whole head quads");
  static constexpr int kNT = kSplit ? G / 2 : (4 * G + 7) / 8;
  static constexpr int kNH = kSplit ? G / 4 : kNT;
  __device__ static int head(int jh, int t) { return kSplit ? 4 * jh + t : 2 * jh + (t >> 1); }
  __device__ static bool owns(int jh, int t) { return kSplit || ((t & 1) == 0 && 2 * jh + (t >> 1) < G); }
  // n (column over all n-tiles) of digit d of head h
  __host__ __device__ static constexpr int column(int h, int d) {
    return kSplit ? 16 * (h >> 2) + 2 * (h & 3) + (d & 1) + 8 * (d >> 1) : 4 * h + d;
  }
};

// p·V records in flight per warp.  With one, p of the record in flight waits in
// registers; with more, each stage also holds its record's p slices (bulk-copied with it).
// 0 (default): two for 2- and 4-bit records, one for 3-bit records (measured: two stages
// took 5% off the GQA p·V and added 5% to the batched 3-bit one; three were slower).
#ifndef PACKKV_PV_STAGES
#define PACKKV_PV_STAGES 0
#endif
// 4-bit records with 8 heads take one: their p slices would make a stage 12.5 KB, and
// with p in registers three CTAs fit per SM (measured on 16 query rows per kv head:
// 69.5 against 88.0 us per call).
constexpr int pv_stages(int bits, int g) {
  return PACKKV_PV_STAGES > 0 ? PACKKV_PV_STAGES : ((bits == 3 || (bits == 4 && g >= 8)) ? 1 : 2);
}

template <int BITS, int G, bool PV>
struct Cfg {
  static constexpr int kRecBytes = raw_record_bytes(BITS);
  static constexpr int kStageRec = kRecBytes;                  // >= every record, staged in one piece
  static constexpr bool kStagedP = PV && pv_stages(BITS, G) > 1;  // p slices [G][128] fp32 after the record
  static constexpr int kStageBytes = kStageRec + (kStagedP ? 512 * G : 0);
  // int8 tensor-core B table: columns n = 4*head + digit (digit 3 = 0), NT n-tiles of 8
  static constexpr int kNT = I8Layout<G>::kNT;
  static constexpr int kNH = I8Layout<G>::kNH;
  static constexpr int kI8Tab = 4 * (64 * kNT + 8) * 4;
  static constexpr int kTableBytes = (kI8Tab + 15) / 16 * 16;
  static constexpr int kSumBytes = PV ? 512 * G : 0;          // p·V: [G][128] channel sums
  static constexpr int kFixed = kTableBytes + kSumBytes;
  static constexpr int kStages0 = (kWarpSmemBudget - kFixed - 64) / kStageBytes;
  static constexpr int kStages = PV ? pv_stages(BITS, G) : (kStages0 > 4 ? 4 : (kStages0 < 1 ? 1 : kStages0));
  static constexpr int kWarpSmem = ((kStages * kStageBytes + kFixed + kStages * 16) + 127) / 128 * 128;
  static_assert(kStageBytes % 16 == 0 && kFixed % 16 == 0, "stage alignment");
};

// Warp-private shared memory: [stages][table][channel sums (p·V)][mbarriers][kinds].
template <int BITS, int G, bool PV>
struct WarpMem {
  using C = Cfg<BITS, G, PV>;
  unsigned char* base;
  __device__ unsigned char* stage(int s) const { return base + s * C::kStageBytes; }
  __device__ unsigned char* fixed() const { return base + C::kStages * C::kStageBytes; }
  __device__ uint32_t* table() const { return reinterpret_cast<uint32_t*>(fixed()); }
  __device__ float* sums() const { return reinterpret_cast<float*>(fixed() + C::kTableBytes); }
  __device__ uint64_t* bar(int s) const { return reinterpret_cast<uint64_t*>(fixed() + C::kFixed) + s; }
  __device__ int* kind(int s) const {
    return reinterpret_cast<int*>(fixed() + C::kFixed + C::kStages * 8) + s;
  }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Warp maximum of non-negative floats, which order like their bit patterns as
// unsigned integers: one warp reduction instruction.
__device__ __forceinline__ float warp_max_nonneg(float x) {
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(x)));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The flat item list of a launch: for every (sequence, head) its packed blocks and then,
// if it has one, its tail.  Uniform batches (NoPlan): every sequence has a.n_blocks
// blocks and a.tail_len tail tokens.  Ragged batches: the RaggedPlan passed with the
// launch gives each sequence's first item and tail length.
struct NoPlan {};

struct Cursor {
  long bh;  // sequence * kv_heads + head
  int j;    // item within the (sequence, head)
  int n;    // items of the (sequence, head)
  int nb;   // packed blocks of the sequence (item j < nb is block j, item nb the tail)
  int tl;   // tail tokens of the sequence
};

template <class A>
__device__ __forceinline__ Cursor cursor_at(const A& a, const NoPlan&, long x) {
  Cursor c;
  c.n = a.items_per_bh;
  c.nb = a.n_blocks;
  c.tl = a.tail_len;
  c.bh = x / c.n;
  c.j = (int)(x % c.n);
  return c;
}

template <class A>
__device__ __forceinline__ Cursor cursor_at(const A& a, const RaggedPlan& p, long x) {
  int lo = 0, hi = a.batch;  // the last sequence whose first item is <= x has items
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.base[mid] <= x) lo = mid; else hi = mid;
  }
  Cursor c;
  c.n = (p.base[lo + 1] - p.base[lo]) / a.kv_heads;
  c.tl = p.tail[lo];
  c.nb = c.n - (c.tl > 0 ? 1 : 0);
  const long r = x - p.base[lo];
  c.bh = (long)lo * a.kv_heads + r / c.n;
  c.j = (int)(r % c.n);
  return c;
}

template <class A>
__device__ __forceinline__ void cursor_next(const A& a, const NoPlan&, Cursor& c) {
  if (++c.j == c.n) {
    c.j = 0;
    ++c.bh;
  }
}

template <class A>
__device__ __forceinline__ void cursor_next(const A& a, const RaggedPlan& p, Cursor& c) {
  if (++c.j < c.n) return;
  c.j = 0;
  ++c.bh;
  if (c.bh % a.kv_heads == 0) {  // the next sequence that has items
    int b = (int)(c.bh / a.kv_heads);
    while (b < a.batch && p.base[b + 1] == p.base[b]) ++b;
    if (b < a.batch) {
      c.n = (p.base[b + 1] - p.base[b]) / a.kv_heads;
      c.tl = p.tail[b];
      c.nb = c.n - (c.tl > 0 ? 1 : 0);
    }
    c.bh = (long)b * a.kv_heads;
  }
}

// Items [first, first + n) of (sequence, head) row bh (n = 0: the row has none).
template <class A>
__device__ __forceinline__ void row_items(const A& a, const NoPlan&, long bh, long* first, long* n) {
  *first = bh * a.items_per_bh;
  *n = a.items_per_bh;
}

template <class A>
__device__ __forceinline__ void row_items(const A& a, const RaggedPlan& p, long bh, long* first, long* n) {
  const long b = bh / a.kv_heads, h = bh % a.kv_heads;
  *n = (p.base[b + 1] - p.base[b]) / a.kv_heads;
  *first = p.base[b] + h * *n;
}

// Row of query head hd of (sequence b, kv head h) in q, scores, p and out: a launch
// serves `group` of the g_total query heads of each kv head, from g_off on.
template <class A>
__device__ __forceinline__ size_t head_row(const A& a, long b, long h, int hd) {
  return ((size_t)b * a.kv_heads + h) * a.g_total + a.g_off + hd;
}

// Index entry {offset16, length16} of block j of row bh: through the block table if the
// cache has one (a physical block outside the index reads as an invalid entry).
template <class A>
__device__ __forceinline__ uint2 block_entry(const A& a, long bh, int j) {
  size_t at;
  if (a.block_table == nullptr) {
    at = (size_t)bh * a.max_blocks + j;
  } else {
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    const int p = a.block_table[(size_t)b * a.max_blocks + j];
    if (p < 0 || (long)p >= (long)a.batch * a.max_blocks) return make_uint2(0xFFFFFFFFu, 0u);
    at = ((size_t)(p / a.max_blocks) * a.kv_heads + h) * a.max_blocks + p % a.max_blocks;
  }
  return *reinterpret_cast<const uint2*>(a.index + at * 2);
}

// Index entries {offset16, length16} of 32 consecutive items of a warp's range, one
// per lane ({0, 0} for a tail item or past the range), loaded with one coalesced
// load (uniform batches without a block table); any lane reads the entry of any item of
// the window by shuffle.
struct EntryWindow {
  long base;  // first item of the window
  uint2 ent;  // entry of item base + lane
  template <class A, class Plan>
  __device__ void load(const A& a, const Plan& plan, long first, long hi, int lane) {
    base = first;
    ent = make_uint2(0u, 0u);
    const long item = first + lane;
    if (item < hi) {
      const Cursor c = cursor_at(a, plan, item);
      if (c.j < c.nb) ent = block_entry(a, c.bh, c.j);
    }
  }
  // Whole warp; base <= item < base + 32.
  __device__ uint2 get(long item) const {
    const int src = (int)(item - base);
    return make_uint2(__shfl_sync(0xffffffffu, ent.x, src), __shfl_sync(0xffffffffu, ent.y, src));
  }
};

// Issue the copies of item c with index entry e into stage s of m (whole warp
// participates); m provides stage(s), bar(s) and kind(s).  The kind slot gets the item
// kind in bits 0..7 and the record's length in 16-byte units above.
template <int BITS, int G, bool PV, class Mem>
__device__ __forceinline__ void issue_item(const GemvArgs& a, const Mem& m, const Cursor& c, uint2 e, int s,
                                           int lane) {
  using C = Cfg<BITS, G, PV>;
  int kind = kKindTail;
  uint64_t off16 = 0;
  uint32_t len16 = 0;
  if (c.j < c.nb) {
    off16 = e.x;
    len16 = e.y;
    const bool valid = e.x != 0xFFFFFFFFu && len16 >= 1040 / 16 && len16 * 16u <= (uint32_t)C::kRecBytes &&
                       off16 + len16 <= a.arena16;
    kind = !valid ? kKindInvalid : (len16 * 16u == (uint32_t)C::kRecBytes ? kKindRaw : kKindPacked);
  }
  unsigned char* st = m.stage(s);
  const unsigned char* src = a.arena + off16 * 16;
  const bool with_p = C::kStagedP && (kind == kKindRaw || kind == kKindPacked);
  if (lane == 0) {
    *m.kind(s) = kind | (int)(len16 << 8);  // kind in bits 0..7, record length (16-B units) above
    uint32_t bytes = 0;
    if (kind == kKindRaw) bytes = C::kRecBytes;
    if (kind == kKindPacked) bytes = len16 * 16u;
    if (with_p) bytes += 512u * G;
    fence_async_smem();
    if (bytes)
      mbar_arrive_expect_tx(m.bar(s), bytes);
    else
      mbar_arrive(m.bar(s));
  }
  __syncwarp();
  if (kind == kKindRaw) {
    if (lane == 16) bulk_g2s(st, src, C::kRecBytes, m.bar(s));
  } else if (kind == kKindPacked) {
    if (lane == 16) bulk_g2s(st, src, len16 * 16u, m.bar(s));
  }
  if (with_p && lane < G) {  // the record's p slices: 128 fp32 of each query head
    const long b = c.bh / a.kv_heads, h = c.bh % a.kv_heads;
    const float* prow = a.p + head_row(a, b, h, lane) * a.ld + (size_t)c.j * 128;
    bulk_g2s(st + C::kStageRec + 512 * lane, prow, 512u, m.bar(s));
  }
}

// After a wait gave up: waits, bounded, for the warp's other copies in flight
// (items x+1 .. prod-1) so that none lands after the warp has exited.
template <int BITS, int G, bool PV>
__device__ void drain_stages(const WarpMem<BITS, G, PV>& m, uint32_t phases, int s, long x, long prod,
                             uint64_t* ctrl) {
  using C = Cfg<BITS, G, PV>;
  for (long i = x + 1; i < prod; ++i) {
    const int si = (int)((s + (i - x)) % C::kStages);
    mbar_wait_bounded(m.bar(si), (phases >> si) & 1u, ctrl);
  }
}

// ----------------------------------------------------------------------------
// 8-bit integer tensor-core decode of raw records (packed-cache format v1, section 4)
// ----------------------------------------------------------------------------
// D(16x8, s32) += A(16x32, u8) * B(32x8, s8): exact integer products and sums.
__device__ __forceinline__ void imma16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The low bytes of four floats of the form r + 1.5*2^23 (r an integer, |r| <= 127):
// the two's-complement bytes of r, packed in order.
__device__ __forceinline__ uint32_t pack4(float2 lo, float2 hi) {
  const uint32_t x0 = __float_as_uint(lo.x), x1 = __float_as_uint(lo.y);
  const uint32_t x2 = __float_as_uint(hi.x), x3 = __float_as_uint(hi.y);
  return __byte_perm(__byte_perm(x0, x1, 0x0040), __byte_perm(x2, x3, 0x0040), 0x5410);
}

// Word of the int8 B table holding B[k = 32*kap + 16*kh + 4*t .. +3][n], read by lane
// 4*(n%8) + t as b_kh of n-tile n/8; a lane's words for one k-step are consecutive.
template <int NT>
__device__ __forceinline__ int i8tab_word(int kap, int kh, int t, int n) {
  return kap * (64 * NT + 8) + (4 * (n & 7) + t) * 2 * NT + kh * NT + (n >> 3);
}

// B table of the int8 products for one record: lane holds x[head][i] for k = 4*lane + i
// (channel for q·Kᵀ, storage slot for p·V).  Per head f = 127 / max|x| and
// y = x*f = d0 + d1/128 + d2/16384 with integer digits |d0| <= 127, |d1|, |d2| <= 64
// (each the rounding of the remainder so far, so |y - sum| <= 2^-15); digit i goes to
// column I8Layout<G>::column(head, i), digit 3 and absent heads are zero.  Returns
// 1/f per head.
template <int G, int NT>
__device__ __forceinline__ void build_i8tab(uint32_t* tab, const float (&x)[G][4], float (&invf)[G], int lane) {
  using L = I8Layout<G>;
  static_assert(NT == L::kNT, "n-tiles of the layout");
  constexpr int kHeads = L::kSplit ? G : 2 * NT;  // heads with columns (absent ones zero)
  const int kap = lane >> 3, kh = (lane >> 2) & 1, t = lane & 3;
  const float2 R = make_float2(kRound, kRound), nR = make_float2(-kRound, -kRound);
  const float2 k128 = make_float2(128.f, 128.f);
#pragma unroll
  for (int hd = 0; hd < kHeads; ++hd) {
    uint32_t w0 = 0u, w1 = 0u, w2 = 0u;
    if (hd < G) {
      const int h = hd < G ? hd : 0;
      const float mx =
          warp_max_nonneg(fmaxf(fmaxf(fabsf(x[h][0]), fabsf(x[h][1])), fmaxf(fabsf(x[h][2]), fabsf(x[h][3]))));
      // |y| <= 127 (the quotient is within 2 ulp); a head whose values are all below
      // 1e-30 gets zero digits (its products are negligible), so f stays finite
      const bool nz = mx > 1e-30f;
      const float f = nz ? __fdividef(127.f, mx) : 0.f;
      invf[h] = nz ? __fdividef(mx, 127.f) : 0.f;
      const float2 m128 = make_float2(-128.f, -128.f);
      float2 t0[2], t1[2], t2[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float2 y = __fmul2_rn(make_float2(x[h][2 * q], x[h][2 * q + 1]), make_float2(f, f));
        t0[q] = __fadd2_rn(y, R);                                          // low byte: d0 = rint(y)
        const float2 r1 = __ffma2_rn(__fadd2_rn(t0[q], nR), m128, __fmul2_rn(y, k128));  // 128(y - d0), exact
        t1[q] = __fadd2_rn(r1, R);                                         // low byte: d1 = rint(r1)
        const float2 r2 = __ffma2_rn(__fadd2_rn(t1[q], nR), m128, __fmul2_rn(r1, k128));  // 128(r1 - d1), exact
        t2[q] = __fadd2_rn(r2, R);                                         // low byte: d2 = rint(r2)
      }
      w0 = pack4(t0[0], t0[1]);
      w1 = pack4(t1[0], t1[1]);
      w2 = pack4(t2[0], t2[1]);
    }
    tab[i8tab_word<NT>(kap, kh, t, L::column(hd, 0))] = w0;
    tab[i8tab_word<NT>(kap, kh, t, L::column(hd, 1))] = w1;
    tab[i8tab_word<NT>(kap, kh, t, L::column(hd, 2))] = w2;
    tab[i8tab_word<NT>(kap, kh, t, L::column(hd, 3))] = 0u;
  }
}

// B fragments of this lane: bf[kap][j] = {b0, b1} of n-tile j at k-step kap.
template <int NT>
__device__ __forceinline__ void load_i8frags(const uint32_t* tab, uint32_t (&bf)[4][NT][2], int lane) {
#pragma unroll
  for (int kap = 0; kap < 4; ++kap) {
    const uint32_t* p = tab + kap * (64 * NT + 8) + lane * 2 * NT;  // [kh][j] words
    if constexpr (NT == 1) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      bf[kap][0][0] = v.x;
      bf[kap][0][1] = v.y;
    } else {
#pragma unroll
      for (int q = 0; q < NT / 2; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(p + 4 * q);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int idx = 4 * q + r, kh = idx / NT, j = idx % NT;
          bf[kap][j][kh] = w4[r];
        }
      }
    }
  }
}

// Accumulators start at the bit pattern of 1.5*2^23 (kRoundBits): an accumulated
// integer D (|D| < 2^22) then reads as the float 1.5*2^23 + D, and
// fmaf(that, w, -w*1.5*2^23) is w*D exactly for a power of two w; further weighted
// digits are chained on with one rounding each.

// Digit weights of a paired-layout thread: even t holds digits 0, 1 (1, 2^-7), odd t
// digit 2 and the zero column (2^-14, 0); c = -(w0 + w1) * 1.5*2^23 (exact).
struct PairW {
  float w0, w1, c;
};
__device__ __forceinline__ PairW pair_weights(int t) {
  const float w0 = (t & 1) ? 1.f / 16384.f : 1.f, w1 = (t & 1) ? 0.f : 1.f / 128.f;
  return {w0, w1, -(w0 + w1) * kRound};
}

// One row of a paired-layout tile (accumulators x0, x1 of columns 2t, 2t + 1): this
// thread's digit terms, before the shuffle join and the row weight.
__device__ __forceinline__ float pair_row(int x0, int x1, const PairW& w) {
  return fmaf(__int_as_float(x1), w.w1, fmaf(__int_as_float(x0), w.w0, w.c));
}

// One row of a split-layout head: digits 0, 1 (x0, x1 of n-tile 2i) and 2 (x2 of
// n-tile 2i + 1) joined, times the row weight u (a power of two).  The first product
// cancels all three offsets, so the running value stays below 2^23 * u.
__device__ __forceinline__ float split_row(int x0, int x1, int x2, float u) {
  constexpr float c = -kRound * (1.f + 1.f / 128.f + 1.f / 16384.f);  // exact: 16 significant bits
  const float v = fmaf(__int_as_float(x0), u, c * u);
  return fmaf(__int_as_float(x2), u * (1.f / 16384.f), fmaf(__int_as_float(x1), u * (1.f / 128.f), v));
}

// The rows of row tile T for every accumulator set jh: emit(T, jh, lo, hi) with the
// values of rows g (lo) and g + 8 (hi), digits joined, valid where
// I8Layout<G>::owns(jh, t).  d: the tile's accumulators over all n-tiles, whose A
// fields carried the powers of two 1/ug (row g) and 1/uh (row g + 8).
template <int G, class Emit>
__device__ __forceinline__ void emit_tile(int T, const int (&d)[I8Layout<G>::kNT][4], float ug, float uh,
                                          const PairW& w, Emit& emit) {
  using L = I8Layout<G>;
  if constexpr (L::kSplit) {
#pragma unroll
    for (int jh = 0; jh < L::kNH; ++jh)
      emit(T, jh, split_row(d[2 * jh][0], d[2 * jh][1], d[2 * jh + 1][0], ug),
           split_row(d[2 * jh][2], d[2 * jh][3], d[2 * jh + 1][2], uh));
  } else {
#pragma unroll
    for (int j = 0; j < L::kNT; ++j) {
      float lo = pair_row(d[j][0], d[j][1], w), hi = pair_row(d[j][2], d[j][3], w);
      lo += __shfl_down_sync(0xffffffffu, lo, 1);
      hi += __shfl_down_sync(0xffffffffu, hi, 1);
      emit(T, j, lo * ug, hi * uh);
    }
  }
}

// As emit_tile for a 3-bit record's two planes: bits 0-1 (dl, row weights ulg, ulh) and
// bit 2 (dh, row weights uhg, uhh, which include the bit's weight 4).
template <int G, class Emit>
__device__ __forceinline__ void emit_tile2(int T, const int (&dl)[I8Layout<G>::kNT][4],
                                           const int (&dh)[I8Layout<G>::kNT][4], float ulg, float ulh, float uhg,
                                           float uhh, const PairW& w, Emit& emit) {
  using L = I8Layout<G>;
  if constexpr (L::kSplit) {
#pragma unroll
    for (int jh = 0; jh < L::kNH; ++jh) {
      const int a = 2 * jh, b = 2 * jh + 1;
      emit(T, jh,
           split_row(dl[a][0], dl[a][1], dl[b][0], ulg) + split_row(dh[a][0], dh[a][1], dh[b][0], uhg),
           split_row(dl[a][2], dl[a][3], dl[b][2], ulh) + split_row(dh[a][2], dh[a][3], dh[b][2], uhh));
    }
  } else {
#pragma unroll
    for (int j = 0; j < L::kNT; ++j) {
      float lo = fmaf(pair_row(dh[j][0], dh[j][1], w), uhg / ulg, pair_row(dl[j][0], dl[j][1], w));
      float hi = fmaf(pair_row(dh[j][2], dh[j][3], w), uhh / ulh, pair_row(dl[j][2], dl[j][3], w));
      lo += __shfl_down_sync(0xffffffffu, lo, 1);
      hi += __shfl_down_sync(0xffffffffu, hi, 1);
      emit(T, j, lo * ulg, hi * ulh);
    }
  }
}

// Selects the value of a run-time head index from a register array.
template <int G>
__device__ __forceinline__ float head_sel(const float (&x)[G], int head) {
  float r = 0.f;
#pragma unroll
  for (int hd = 0; hd < G; ++hd)
    if (head == hd) r = x[hd];
  return r;
}

// A registers of one row tile from its two fragment words (k halves kh = 0, 1).
// b = 4: row g + 8 is the high nibbles (x16).  Row g is the low nibbles, or with
// kWholeBytes the whole bytes, i.e. its codes plus the high nibbles x16: both rows
// meet the same B values, so the surplus is exactly row g + 8's accumulator,
// subtracted after the k-steps (unmask4), and a word costs one AND instead of two.
template <bool kWholeBytes>
__device__ __forceinline__ void afrag4(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  a[0] = kWholeBytes ? w0 : w0 & 0x0F0F0F0Fu;
  a[1] = w0 & 0xF0F0F0F0u;
  a[2] = kWholeBytes ? w1 : w1 & 0x0F0F0F0Fu;
  a[3] = w1 & 0xF0F0F0F0u;
}

// Row g of an afrag4 tile: its accumulators minus row g + 8's (columns 2t, 2t + 1),
// keeping the 1.5*2^23 offset.  Exact: |sum over k of byte * b| <= 128*255*127 < 2^22.
__device__ __forceinline__ void unmask4(int (&d)[4]) {
  d[0] = d[0] - d[2] + kRoundBits;
  d[1] = d[1] - d[3] + kRoundBits;
}

// b = 2: even tile rows g (x1), g + 8 (x4); odd tile rows g (x16), g + 8 (x64).
__device__ __forceinline__ void afrag2(uint32_t w0, uint32_t w1, uint32_t (&ae)[4], uint32_t (&ao)[4]) {
  ae[0] = w0 & 0x03030303u;
  ae[1] = w0 & 0x0C0C0C0Cu;
  ae[2] = w1 & 0x03030303u;
  ae[3] = w1 & 0x0C0C0C0Cu;
  ao[0] = w0 & 0x30303030u;
  ao[1] = w0 & 0xC0C0C0C0u;
  ao[2] = w1 & 0x30303030u;
  ao[3] = w1 & 0xC0C0C0C0u;
}

// The bit-2 plane of a 3-bit record: tile T's rows g and g + 8 sit at bit 2(T mod 4)
// and 2(T mod 4) + 1 of every byte; A registers from the plane's two words (kh 0, 1).
template <int TQ>
__device__ __forceinline__ void afrag1(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  constexpr uint32_t lo = 0x01010101u << (2 * TQ), hi = 0x02020202u << (2 * TQ);
  a[0] = w0 & lo;
  a[1] = w0 & hi;
  a[2] = w1 & lo;
  a[3] = w1 & hi;
}

// Runs the tensor-core product of one raw record: for every row tile T (16 rows) and
// accumulator set jh calls emit(T, jh, lo, hi) with the values of rows g (lo) and
// g + 8 (hi) for head I8Layout<G>::head(jh, t), digits joined (see emit_tile).  Rows
// are slots (q·Kᵀ, K record) or channels (p·V, V record).
template <int BITS, int G, bool kWholeBytes, class Emit>
__device__ __forceinline__ void i8_product(const unsigned char* st,
                                           const uint32_t (&bf)[4][I8Layout<G>::kNT][2], int lane, Emit&& emit) {
  constexpr int NT = I8Layout<G>::kNT;
  const uint4* words = reinterpret_cast<const uint4*>(st + kRawWordOffset);
  const PairW pw = pair_weights(lane & 3);
  if constexpr (BITS == 4) {
#pragma unroll
    for (int T = 0; T < 8; ++T) {
      const uint4 wa = words[(T * 2) * 32 + lane], wb = words[(T * 2 + 1) * 32 + lane];
      // k-step kap: words (kh 0, kh 1) = (wa.x, wa.y), (wa.z, wa.w), (wb.x, wb.y), (wb.z, wb.w)
      const uint32_t w[4][2] = {{wa.x, wa.y}, {wa.z, wa.w}, {wb.x, wb.y}, {wb.z, wb.w}};
      int d[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = kRoundBits;
#pragma unroll
      for (int kap = 0; kap < 4; ++kap) {
        uint32_t a[4];
        afrag4<kWholeBytes>(w[kap][0], w[kap][1], a);
#pragma unroll
        for (int j = 0; j < NT; ++j) imma16832(d[j], a, bf[kap][j][0], bf[kap][j][1]);
      }
      if (kWholeBytes) {
#pragma unroll
        for (int j = 0; j < NT; ++j) unmask4(d[j]);
      }
      emit_tile<G>(T, d, 1.f, 1.f / 16.f, pw, emit);  // low nibbles x1, high nibbles x16
    }
  } else if constexpr (BITS == 2) {
#pragma unroll
    for (int P = 0; P < 4; ++P) {  // tile pairs
      const uint4 wa = words[(P * 2) * 32 + lane], wb = words[(P * 2 + 1) * 32 + lane];
      const uint32_t w[4][2] = {{wa.x, wa.y}, {wa.z, wa.w}, {wb.x, wb.y}, {wb.z, wb.w}};
      int de[NT][4], dd[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) de[j][i] = dd[j][i] = kRoundBits;
#pragma unroll
      for (int kap = 0; kap < 4; ++kap) {
        uint32_t ae[4], ao[4];
        afrag2(w[kap][0], w[kap][1], ae, ao);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          imma16832(de[j], ae, bf[kap][j][0], bf[kap][j][1]);
          imma16832(dd[j], ao, bf[kap][j][0], bf[kap][j][1]);
        }
      }
      emit_tile<G>(2 * P, de, 1.f, 0.25f, pw, emit);               // even tile: x1, x4
      emit_tile<G>(2 * P + 1, dd, 1.f / 16.f, 1.f / 64.f, pw, emit);  // odd tile: x16, x64
    }
  } else {
    const uint4* hwords = words + 1024 / 4;  // bit-2 plane
#pragma unroll
    for (int Q = 0; Q < 2; ++Q) {  // tile quads of the bit-2 plane
      const uint4 ha = hwords[(Q * 2) * 32 + lane], hb = hwords[(Q * 2 + 1) * 32 + lane];
      const uint32_t hw[4][2] = {{ha.x, ha.y}, {ha.z, ha.w}, {hb.x, hb.y}, {hb.z, hb.w}};
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {  // tile pairs 2Q + pp: tiles 4Q + 2pp, 4Q + 2pp + 1
        const int P = 2 * Q + pp;
        const uint4 wa = words[(P * 2) * 32 + lane], wb = words[(P * 2 + 1) * 32 + lane];
        const uint32_t w[4][2] = {{wa.x, wa.y}, {wa.z, wa.w}, {wb.x, wb.y}, {wb.z, wb.w}};
        int le[NT][4], lo_[NT][4], he[NT][4], ho[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) le[j][i] = lo_[j][i] = he[j][i] = ho[j][i] = kRoundBits;
#pragma unroll
        for (int kap = 0; kap < 4; ++kap) {
          uint32_t ae[4], ao[4], be[4], bo[4];
          afrag2(w[kap][0], w[kap][1], ae, ao);
          if (pp == 0) {
            afrag1<0>(hw[kap][0], hw[kap][1], be);
            afrag1<1>(hw[kap][0], hw[kap][1], bo);
          } else {
            afrag1<2>(hw[kap][0], hw[kap][1], be);
            afrag1<3>(hw[kap][0], hw[kap][1], bo);
          }
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            imma16832(le[j], ae, bf[kap][j][0], bf[kap][j][1]);
            imma16832(lo_[j], ao, bf[kap][j][0], bf[kap][j][1]);
            imma16832(he[j], be, bf[kap][j][0], bf[kap][j][1]);
            imma16832(ho[j], bo, bf[kap][j][0], bf[kap][j][1]);
          }
        }
        // bit 2 weighs 4; tile 4Q + s (s = 2pp, 2pp+1) carries 2^(2s) (row g), 2^(2s+1) (row g+8)
        const float e0 = 4.f / float(1 << (4 * pp)), e1 = 4.f / float(1 << (4 * pp + 2));
        emit_tile2<G>(2 * P, le, he, 1.f, 0.25f, e0, e0 * 0.5f, pw, emit);
        emit_tile2<G>(2 * P + 1, lo_, ho, 1.f / 16.f, 1.f / 64.f, e1, e1 * 0.5f, pw, emit);
      }
    }
  }
}

// q·Kᵀ of one raw K record: scores of all 128 slots for the G heads.
template <int BITS, int G>
__device__ __forceinline__ void qk_i8(const unsigned char* st, const uint32_t* tab, const float (&cst)[G],
                                      const float (&invf)[G], float* sblk, long ld, float scale, int lane) {
  using L = I8Layout<G>;
  const int g = lane >> 2, t = lane & 3;
  uint32_t bf[4][L::kNT][2];
  load_i8frags<L::kNT>(tab, bf, lane);
  // per accumulator set: this thread's head with the score scale folded in
  float sf[L::kNH], sc[L::kNH];
#pragma unroll
  for (int jh = 0; jh < L::kNH; ++jh) {
    const int head = L::head(jh, t);
    sf[jh] = scale * head_sel<G>(invf, head);
    sc[jh] = scale * head_sel<G>(cst, head);
  }
  i8_product<BITS, G, true>(st, bf, lane, [&](int T, int jh, float lo, float hi) {
    if (L::owns(jh, t)) {
      float* dst = sblk + L::head(jh, t) * ld + 16 * T + g;
      dst[0] = fmaf(lo, sf[jh], sc[jh]);
      dst[8] = fmaf(hi, sf[jh], sc[jh]);
    }
  });
}

// p·V of one raw V record: adds sum_slots p'*code into the accumulators of channels
// 16T + g (acc_lo) and 16T + g + 8 (acc_hi) of head I8Layout<G>::head(jh, t).
template <int BITS, int G>
__device__ __forceinline__ void pv_i8(const unsigned char* st, const uint32_t* tab, const float (&invf)[G],
                                      float (&acc_lo)[I8Layout<G>::kNH][8], float (&acc_hi)[I8Layout<G>::kNH][8],
                                      int lane) {
  using L = I8Layout<G>;
  const int t = lane & 3;
  uint32_t bf[4][L::kNT][2];
  load_i8frags<L::kNT>(tab, bf, lane);
  float f_t[L::kNH];
#pragma unroll
  for (int jh = 0; jh < L::kNH; ++jh) f_t[jh] = head_sel<G>(invf, L::head(jh, t));
  i8_product<BITS, G, false>(st, bf, lane, [&](int T, int jh, float lo, float hi) {
    acc_lo[jh][T] = fmaf(lo, f_t[jh], acc_lo[jh][T]);
    acc_hi[jh][T] = fmaf(hi, f_t[jh], acc_hi[jh][T]);
  });
}

// ----------------------------------------------------------------------------
// Compressed records on the 8-bit integer tensor cores
// ----------------------------------------------------------------------------
// A compressed unit (pack group g, channel c) holds the 32 offsets of its slots in w
// words: power-of-two slices of 4, 2 and 1 bits (packed-cache format v1, section 3).
// A tensor-core register takes four codes, and lanes must decode with the same
// instructions whatever the widths of their units:
//  * q·Kᵀ (contraction over channels): a register holds four channels of one slot, so
//    four units are joined per register.  The units of a group are sorted by width
//    (classes 4, 3, 2, 1; a unit of width 0 carries only its base and is left out), each
//    class padded with dummy units to a multiple of 16, so every run of 16 sorted units
//    has one width and is one k half (16 channels) of an m16n8k32 product.  Lane (g8, t)
//    takes the channels at run positions 4t..4t+3 and slots 4g8..4g8+3 of the group (rows
//    g8 and g8 + 8 of the group's two 16-slot tiles), joins the four units' slot runs with
//    byte permutes and separates the codes with masks.  The B operand (q' digits, in
//    natural channel order in the table of build_i8tab) is gathered through the sort.
//  * p·V (contraction over slots, along the units): natural channel order, every slice
//    kind decoded by every lane and masked by the unit's width (pv_packed_nat).
// The prologue reads the record's meta into registers, after which bytes [0, 1040) of
// the stage (header, params, meta) are free for descriptors.  q·Kᵀ: sorted descriptors
// (word start | tag << 16); words [1024, 1040) are zeroed and a dummy unit starts there
// (word index -4 of the word area), so it decodes to zero codes.
constexpr int kZeroUnitStart = -4;

// Reads and checks a staged compressed record: widths <= BITS, total_words = the sum of
// the widths, and a record length that matches it (so that every word a unit of the
// record can name lies inside the staged bytes).  m4[g] = the meta bytes of this lane's
// channels 4*lane .. 4*lane + 3 in group g.  Whole warp; returns the same verdict to all.
template <int BITS>
__device__ __forceinline__ bool packed_prologue(unsigned char* st, uint32_t len, uint32_t (&m4)[4], int lane) {
  const uint32_t* meta = reinterpret_cast<const uint32_t*>(st + kMetaOffset);
  uint32_t wsum = 0u, bad = 0u;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    m4[g] = meta[g * 32 + lane];
    const uint32_t w = (m4[g] >> 4) & 0x0F0F0F0Fu;
    wsum = __dp4a(w, 0x01010101u, wsum);
    bad |= (w + (0x7Fu - BITS) * 0x01010101u) & 0x80808080u;  // a width above BITS sets bit 7
  }
  int tot = (int)wsum;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  const uint32_t total_words = reinterpret_cast<const uint32_t*>(st)[3];
  const bool ok = !__any_sync(0xffffffffu, bad != 0u) && (uint32_t)tot == total_words &&
                  ((1040u + 4u * (uint32_t)tot + 15u) & ~15u) == len;
  __syncwarp();  // every lane has read the header and meta: [0, 1040) may be overwritten
  if (lane < 4) reinterpret_cast<uint32_t*>(st + 1024)[lane] = 0u;
  return ok;
}

// Run positions of one group after the sort: nblk runs of 16, classes 4, 3, 2 end
// (padded) at end4, end3, end2 and class 1 fills the rest.
struct SortedGroup {
  int nblk, end4, end3, end2;
  __device__ int width(int blk) const {
    const int p = 16 * blk;
    return p < end4 ? 4 : (p < end3 ? 3 : (p < end2 ? 2 : 1));
  }
};

// Sorts the units of one group by width into desc[] (whole warp).  m4: this lane's meta
// bytes (channels 4*lane + i); wbase: word index where the group starts (advanced by the
// group's words); tag(c): the descriptor's high half for channel c.  Counting sort: a
// packed per-class count (byte 4 - w for width w) is scanned over the warp together with
// the widths (word starts in channel order).
template <class Tag>
__device__ __forceinline__ SortedGroup sort_group(uint32_t m4, int& wbase, uint32_t* desc, uint32_t dummy, Tag tag,
                                                  int lane) {
  uint32_t w[4];
  int ls = 0;
  uint32_t cnt = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = (m4 >> (8 * i + 4)) & 15u;
    ls += (int)w[i];
    cnt += w[i] ? 1u << (32u - 8u * w[i]) : 0u;
  }
  int incl = ls;
  uint32_t cincl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    const uint32_t cy = __shfl_up_sync(0xffffffffu, cincl, o);
    if (lane >= o) {
      incl += y;
      cincl += cy;
    }
  }
  const int gtot = __shfl_sync(0xffffffffu, incl, 31);
  const uint32_t ctot = __shfl_sync(0xffffffffu, cincl, 31);
  int s = wbase + incl - ls;
  wbase += gtot;
  const uint32_t n0 = ctot & 255u, n1 = (ctot >> 8) & 255u, n2 = (ctot >> 16) & 255u, n3 = ctot >> 24;
  const uint32_t p0 = (n0 + 15u) & ~15u, p1 = (n1 + 15u) & ~15u, p2 = (n2 + 15u) & ~15u, p3 = (n3 + 15u) & ~15u;
  const uint32_t b1 = p0, b2 = b1 + p1, b3 = b2 + p2;
  // per class byte: the position of this lane's next unit of that class (<= 187: no carries)
  uint32_t at = ((b1 << 8) | (b2 << 16) | (b3 << 24)) + (cincl - cnt);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (w[i]) {
      const uint32_t sh = 32u - 8u * w[i];
      desc[(at >> sh) & 255u] = ((uint32_t)s & 0xFFFFu) | (tag(4 * lane + i) << 16);
      at += 1u << sh;
    }
    s += (int)w[i];
  }
  // dummies fill each class up to its padded size
  if ((uint32_t)lane < p0 - n0) desc[n0 + lane] = dummy;
  if ((uint32_t)lane < p1 - n1) desc[b1 + n1 + lane] = dummy;
  if ((uint32_t)lane < p2 - n2) desc[b2 + n2 + lane] = dummy;
  if ((uint32_t)lane < p3 - n3) desc[b3 + n3 + lane] = dummy;
  SortedGroup r;
  r.nblk = (int)((b3 + p3) >> 4);
  r.end4 = (int)b1;
  r.end3 = (int)b2;
  r.end2 = (int)b3;
  return r;
}

__device__ __forceinline__ int desc_start(uint32_t d) { return (int)(int16_t)(d & 0xFFFFu); }

// Exact float of a small unsigned integer (< 2^23): it goes into the mantissa of 2^23.
__device__ __forceinline__ float small_u2f(uint32_t u) { return __uint_as_float(u | 0x4B000000u) - 8388608.f; }

// q·Kᵀ: A registers of one 16-unit run of width W for lane (g8, t): R[i] = the codes of
// slot 4*g8 + i of the four units d (run positions 4t .. 4t+3), one byte per unit.
template <int W>
__device__ __forceinline__ void qk_run(const uint32_t* words, const uint4 d, int g8, uint32_t (&R)[4]) {
  const int s0 = desc_start(d.x), s1 = desc_start(d.y), s2 = desc_start(d.z), s3 = desc_start(d.w);
  if constexpr (W == 4) {
    // slots 4*g8 .. +3: the 16-bit half g8 & 1 of word g8 >> 1 (a nibble per slot)
    const int o = g8 >> 1;
    const uint32_t sel = (g8 & 1) ? 0x7632u : 0x5410u;
    const uint32_t y01 = __byte_perm(words[s0 + o], words[s1 + o], sel);
    const uint32_t y23 = __byte_perm(words[s2 + o], words[s3 + o], sel);
    const uint32_t p0 = __byte_perm(y01, y23, 0x6420u), p1 = __byte_perm(y01, y23, 0x7531u);
    R[0] = p0 & 0x0F0F0F0Fu;
    R[1] = (p0 >> 4) & 0x0F0F0F0Fu;
    R[2] = p1 & 0x0F0F0F0Fu;
    R[3] = (p1 >> 4) & 0x0F0F0F0Fu;
  } else {
    // 2-bit slice: byte g8 & 3 of word g8 >> 1 ... >> 2; 1-bit slice: nibble g8 & 1 of byte g8 >> 1
    uint32_t p2 = 0u, p1 = 0u;
    if constexpr (W == 2 || W == 3) {
      const int o = g8 >> 2;
      const uint32_t b = (uint32_t)(g8 & 3), sel = b | ((b + 4u) << 4);
      const uint32_t y01 = __byte_perm(words[s0 + o], words[s1 + o], sel);
      const uint32_t y23 = __byte_perm(words[s2 + o], words[s3 + o], sel);
      p2 = __byte_perm(y01, y23, 0x5410u);
    }
    if constexpr (W == 1 || W == 3) {
      const int o = W == 3 ? 2 : 0;
      const uint32_t b = (uint32_t)(g8 >> 1), sel = b | ((b + 4u) << 4);
      const uint32_t y01 = __byte_perm(words[s0 + o], words[s1 + o], sel);
      const uint32_t y23 = __byte_perm(words[s2 + o], words[s3 + o], sel);
      p1 = __byte_perm(y01, y23, 0x5410u) >> (4 * (g8 & 1));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t r = 0u;
      if constexpr (W == 2 || W == 3) r = (p2 >> (2 * i)) & 0x03030303u;
      if constexpr (W == 1) r = (p1 >> i) & 0x01010101u;
      if constexpr (W == 3) r |= ((p1 >> i) & 0x01010101u) << 2;
      R[i] = r;
    }
  }
}

// Byte `off` past each of the four units' B-table bases (the descriptors' high halves),
// packed in order.
__device__ __forceinline__ uint32_t gather4(const uint8_t* t8, const uint4 d, int off) {
  const uint32_t x0 = t8[(d.x >> 16) + off], x1 = t8[(d.y >> 16) + off];
  const uint32_t x2 = t8[(d.z >> 16) + off], x3 = t8[(d.w >> 16) + off];
  return __byte_perm(__byte_perm(x0, x1, 0x0040u), __byte_perm(x2, x3, 0x0040u), 0x5410u);
}

// q·Kᵀ of one compressed K record on the tensor cores.  tab: the int8 B table of q'
// (build_i8tab, natural channel order); qv: this lane's q' = q * scale_c for channels
// 4*lane .. +3; cst: sum_c q_c mn_c per head.  Writes the 128 scores of every head:
// scale * (cst + sum_c q'_c base_gc + sum_c q'_c offset).
// Returns false (nothing written) if the record fails the prologue's checks.
template <int BITS, int G>
__device__ __forceinline__ bool qk_packed_tc(unsigned char* st, uint32_t len, const uint32_t* tab,
                                             const float (&qv)[G][4], const float (&cst)[G], const float (&invf)[G],
                                             float* sblk, long ld, float scale, int lane) {
  using L = I8Layout<G>;
  constexpr int NT = L::kNT;
  uint32_t m4[4];
  if (!packed_prologue<BITS>(st, len, m4, lane)) return false;
  const int g8 = lane >> 2, t = lane & 3;
  uint32_t* desc = reinterpret_cast<uint32_t*>(st);
  const uint32_t* words = reinterpret_cast<const uint32_t*>(st + kPackedWordOffset);
  const uint8_t* t8 = reinterpret_cast<const uint8_t*>(tab);
  // byte of channel c's B digits in the table (column n adds 4 * (8 NT (n & 7) + (n >> 3)))
  auto tag = [](int c) -> uint32_t {
    return 4u * (uint32_t)((c >> 5) * (64 * NT + 8) + ((c >> 2) & 3) * 2 * NT + ((c >> 4) & 1) * NT) + (uint32_t)(c & 3);
  };
  const uint32_t dummy = (uint32_t)kZeroUnitStart & 0xFFFFu;
  // base terms of the four groups, sum_c q'_c base_gc, kept in the free stage bytes
  // [768, 1024) (qv is then dead, which keeps the register count of the raw path)
  float* bsm = reinterpret_cast<float*>(st + 768);
#pragma unroll
  for (int g = 0; g < 4; ++g)
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      float part = qv[hd][0] * small_u2f(m4[g] & 15u);
      part = fmaf(qv[hd][1], small_u2f((m4[g] >> 8) & 15u), part);
      part = fmaf(qv[hd][2], small_u2f((m4[g] >> 16) & 15u), part);
      part = fmaf(qv[hd][3], small_u2f((m4[g] >> 24) & 15u), part);
      part = warp_sum(part);
      if (lane == 0) bsm[g * G + hd] = part + cst[hd];
    }
  const PairW pw = pair_weights(t);
  float sf[L::kNH];
#pragma unroll
  for (int jh = 0; jh < L::kNH; ++jh) sf[jh] = scale * head_sel<G>(invf, L::head(jh, t));
  int wbase = 0;
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    __syncwarp();  // the previous group's runs are decoded: desc may be rewritten
    const SortedGroup sg = sort_group(m4[g], wbase, desc, dummy, tag, lane);
    float sc_[L::kNH];
#pragma unroll
    for (int jh = 0; jh < L::kNH; ++jh) sc_[jh] = scale * bsm[g * G + L::head(jh, t)];
    __syncwarp();  // desc of this group written
    int acc[2][NT][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int j = 0; j < NT; ++j) acc[u][j][0] = acc[u][j][1] = acc[u][j][2] = acc[u][j][3] = kRoundBits;
#pragma unroll 1
    for (int blk0 = 0; blk0 < sg.nblk; blk0 += 2) {
      uint32_t R[2][4], bf[2][NT];
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
        const int blk = blk0 + kh;
        if (blk < sg.nblk) {
          const uint4 d = *reinterpret_cast<const uint4*>(desc + 16 * blk + 4 * t);
          switch (sg.width(blk)) {  // warp-uniform
            case 4: qk_run<4>(words, d, g8, R[kh]); break;
            case 3: qk_run<3>(words, d, g8, R[kh]); break;
            case 2: qk_run<2>(words, d, g8, R[kh]); break;
            default: qk_run<1>(words, d, g8, R[kh]); break;
          }
#pragma unroll
          for (int j = 0; j < NT; ++j) bf[kh][j] = gather4(t8, d, 4 * (8 * NT * g8 + j));
        } else {
          R[kh][0] = R[kh][1] = R[kh][2] = R[kh][3] = 0u;
#pragma unroll
          for (int j = 0; j < NT; ++j) bf[kh][j] = 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {  // the group's two tiles: rows g8 / g8 + 8 = slots 4 g8 + 2u / + 1
        const uint32_t a[4] = {R[0][2 * u], R[0][2 * u + 1], R[1][2 * u], R[1][2 * u + 1]};
#pragma unroll
        for (int j = 0; j < NT; ++j) imma16832(acc[u][j], a, bf[0][j], bf[1][j]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      auto emit = [&](int, int jh, float lo, float hi) {
        if (L::owns(jh, t)) {
          float* dst = sblk + L::head(jh, t) * ld + 32 * g + 4 * g8 + 2 * u;
          *reinterpret_cast<float2*>(dst) = make_float2(fmaf(lo, sf[jh], sc_[jh]), fmaf(hi, sf[jh], sc_[jh]));
        }
      };
      emit_tile<G>(u, acc[u], 1.f, 1.f, pw, emit);
    }
  }
  return true;
}

// The fp16 tail (tl tokens, after the sequence's nb blocks) of row bh: scaled scores.
template <int G>
__device__ __forceinline__ void qk_tail(const GemvArgs& a, long bh, int nb, int tl, const float (&qr)[G][4],
                                        float* srow0, int lane) {
  const uint16_t* tail = a.tail + (size_t)bh * 128 * 128;
  for (int t0 = 0; t0 < tl; t0 += 32) {
    float mine[G];
#pragma unroll
    for (int hd = 0; hd < G; ++hd) mine[hd] = 0.f;
    const int tn = min(32, tl - t0);
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
      for (int hd = 0; hd < G; ++hd) srow0[hd * a.ld + (long)nb * 128 + t0 + lane] = a.scale * mine[hd];
    }
  }
}

// p·V k orders: the k position (kh, t, e) of an A or B register of lane t (kh: the
// register's k half, e: its byte) holds
//   slot 8t + 2e + kh  (order A: a 4-bit slice gives a register per mask of word t), or
//   slot t + 8e + 4kh  (order B: 2- and 1-bit slices give a register per shift and mask).

// B fragments of group g in the two k orders, gathered from the int8 B table
// of p' (build_i8tab, natural slot order: byte k & 3 of word i8tab_word(k >> 5,
// (k >> 4) & 1, (k >> 2) & 3, n) holds slot k).  bA/bB[kh][j] for n-tile j.
template <int NT>
__device__ __forceinline__ void pv_group_frags(const uint32_t* tab, int g, int lane, uint32_t (&bA)[2][NT],
                                               uint32_t (&bB)[2][NT]) {
  const int g8 = lane >> 2, t = lane & 3;
  const uint8_t* t8 = reinterpret_cast<const uint8_t*>(tab);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int n = 8 * j + g8;
    // order A: slot 8t + 2e + kh = natural (kh' = t >> 1, t' = 2(t & 1) + (e >> 1), e' = 2(e & 1) + kh)
    const uint32_t w0 = tab[i8tab_word<NT>(g, t >> 1, 2 * (t & 1), n)];
    const uint32_t w1 = tab[i8tab_word<NT>(g, t >> 1, 2 * (t & 1) + 1, n)];
    bA[0][j] = __byte_perm(w0, w1, 0x6420u);
    bA[1][j] = __byte_perm(w0, w1, 0x7531u);
    // order B: slot t + 8e + 4kh = natural (kh' = e >> 1, t' = 2(e & 1) + kh, e' = t)
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const uint32_t x0 = t8[4 * i8tab_word<NT>(g, 0, kh, n) + t], x1 = t8[4 * i8tab_word<NT>(g, 0, 2 + kh, n) + t];
      const uint32_t x2 = t8[4 * i8tab_word<NT>(g, 1, kh, n) + t], x3 = t8[4 * i8tab_word<NT>(g, 1, 2 + kh, n) + t];
      bB[kh][j] = __byte_perm(__byte_perm(x0, x1, 0x0040u), __byte_perm(x2, x3, 0x0040u), 0x5410u);
    }
  }
}

// p·V in natural channel order.  Row tile T = channels 16T .. 16T+15 (the tiles of raw
// records), k-step g = pack group g.  Every lane decodes its two units of a tile with
// the same instructions whatever their widths: a 4-bit slice in k order A,
// the 2- and 1-bit slices and the unit's base in k order B, a slice the unit lacks
// masked to zero.  Two products per tile, one per order, add into the same
// accumulators, so a tile ends with sum_r p'_r (base + offset) of its channels.  No
// sort: every tile's rows are fixed channels.
//
// Descriptor of unit (g, c): group-relative word start | width << 9 | base << 12 (the
// start is at most 127 * 4, the base at most 15); word 64g + 8T + (c & 7) of the stage's
// free bytes holds channel 16T + (c & 7) in its low half and channel 16T + (c & 7) + 8
// in its high half, so a lane reads both of its rows with one load.  The loads do not
// depend on the width (no divergence); a word read past a unit's end still lies in the
// staged record or the stage's slack (a compressed record is at least 16 bytes shorter
// than a raw one) and is masked off.
#ifndef PACKKV_NAT_FRAG_NT
#define PACKKV_NAT_FRAG_NT 2
#endif
__device__ __forceinline__ void pv_nat_unit(const uint32_t* words, int gs, uint32_t dsc, int t, uint32_t& a0,
                                            uint32_t& a1, uint32_t& b0, uint32_t& b1) {
  const int s = gs + (int)(dsc & 511u);
  const uint32_t w = (dsc >> 9) & 7u;
  const uint32_t bb = (dsc >> 12) * 0x01010101u;
  const uint32_t m4 = w == 4u ? 0x0F0F0F0Fu : 0u;
  const uint32_t m2 = (w & 2u) ? 0x03030303u : 0u;
  const uint32_t m1 = (w & 1u) ? 0x01010101u : 0u;
  const uint32_t x4 = words[s + t];  // 4-bit slice: slots 8t .. 8t+7, a nibble each
  const uint32_t x20 = words[s], x21 = words[s + 1];  // 2-bit slice: bits 0-1 of the offsets
  const uint32_t x1 = words[s + (int)(w & 2u)];       // 1-bit slice: bit 0 (width 1) or bit 2 (width 3)
  a0 = x4 & m4;
  a1 = (x4 >> 4) & m4;
  const uint32_t k1 = (w & 2u) ? 4u : 1u;
  const uint32_t y = x1 >> t;  // bit t + 8e + 4kh -> bit 8e (kh = 0) / 8e + 4 (kh = 1)
  b0 = ((__byte_perm(x20, x21, 0x6420u) >> (2 * t)) & m2) + (y & m1) * k1 + bb;
  b1 = ((__byte_perm(x20, x21, 0x7531u) >> (2 * t)) & m2) + ((y >> 4) & m1) * k1 + bb;
}

// p·V of one compressed V record in natural channel order (see pv_nat_unit): adds
// sum_r p'_r code[r][c], digits joined and times invf, into sacc (the warp's [G][128]
// channel sums).  tab: the int8 B table of p' in natural slot order (build_i8tab).
// Returns false (nothing added) if the record fails the prologue's checks.
template <int BITS, int G>
__device__ __forceinline__ bool pv_packed_nat(unsigned char* st, uint32_t len, const uint32_t* tab,
                                              const float (&invf)[G], float* sacc, int lane) {
  using L = I8Layout<G>;
  constexpr int NT = L::kNT;
  constexpr bool kFragRegs = NT <= PACKKV_NAT_FRAG_NT;  // B fragments of all four groups in registers
  uint32_t m4[4];
  if (!packed_prologue<BITS>(st, len, m4, lane)) return false;
  const int g8 = lane >> 2, t = lane & 3;
  // word starts: lane sums of the widths, two groups per 16-bit half, scanned over the warp
  uint32_t ls[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) ls[g] = __dp4a((m4[g] >> 4) & 0x0F0F0F0Fu, 0x01010101u, 0u);
  uint32_t inc0 = ls[0] | (ls[1] << 16), inc1 = ls[2] | (ls[3] << 16);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
    if (lane >= o) {
      inc0 += y0;
      inc1 += y1;
    }
  }
  const uint32_t tot0 = __shfl_sync(0xffffffffu, inc0, 31), tot1 = __shfl_sync(0xffffffffu, inc1, 31);
  const int gs1 = (int)(tot0 & 0xFFFFu), gs2 = gs1 + (int)(tot0 >> 16), gs3 = gs2 + (int)(tot1 & 0xFFFFu);
  const uint32_t ex0 = inc0 - (ls[0] | (ls[1] << 16)), ex1 = inc1 - (ls[2] | (ls[3] << 16));
  const uint32_t ex[4] = {ex0 & 0xFFFFu, ex0 >> 16, ex1 & 0xFFFFu, ex1 >> 16};
  uint16_t* d16 = reinterpret_cast<uint16_t*>(st);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t rel = ex[g];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t mb = (m4[g] >> (8 * i)) & 0xFFu;  // base | width << 4
      const uint32_t w = mb >> 4;
      d16[2 * (64 * g + 8 * (lane >> 2) + 4 * (lane & 1) + i) + ((lane >> 1) & 1)] =
          (uint16_t)(rel | (w << 9) | ((mb & 15u) << 12));
      rel += w;
    }
  }
  uint32_t bA[kFragRegs ? 4 : 1][2][NT], bB[kFragRegs ? 4 : 1][2][NT];
  if constexpr (kFragRegs) {
#pragma unroll
    for (int g = 0; g < 4; ++g) pv_group_frags<NT>(tab, g, lane, bA[g], bB[g]);
  }
  __syncwarp();  // descriptors written
  const uint32_t* words = reinterpret_cast<const uint32_t*>(st + kPackedWordOffset);
  const uint32_t* dsc = reinterpret_cast<const uint32_t*>(st) + g8;
  const PairW pw = pair_weights(t);
  float f_t[L::kNH];
#pragma unroll
  for (int jh = 0; jh < L::kNH; ++jh) f_t[jh] = head_sel<G>(invf, L::head(jh, t));
#pragma unroll 1
  for (int T = 0; T < 8; ++T) {
    int d[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = kRoundBits;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t x = dsc[64 * g + 8 * T];
      const int gs = g == 0 ? 0 : (g == 1 ? gs1 : (g == 2 ? gs2 : gs3));
      uint32_t aA[4], aB[4];  // rows g8 / g8 + 8 at kh 0, then kh 1
      pv_nat_unit(words, gs, x & 0xFFFFu, t, aA[0], aA[2], aB[0], aB[2]);
      pv_nat_unit(words, gs, x >> 16, t, aA[1], aA[3], aB[1], aB[3]);
      const int gi = kFragRegs ? g : 0;
      if constexpr (!kFragRegs) pv_group_frags<NT>(tab, g, lane, bA[0], bB[0]);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        imma16832(d[j], aA, bA[gi][0][j], bA[gi][1][j]);
        imma16832(d[j], aB, bB[gi][0][j], bB[gi][1][j]);
      }
    }
    auto emit = [&](int TT, int jh, float lo, float hi) {
      if (L::owns(jh, t)) {
        float* row = sacc + L::head(jh, t) * 128 + 16 * TT + g8;
        row[0] = fmaf(lo, f_t[jh], row[0]);
        row[8] = fmaf(hi, f_t[jh], row[8]);
      }
    };
    emit_tile<G>(T, d, 1.f, 1.f, pw, emit);
  }
  __syncwarp();  // sums added before other lanes read or add them
  return true;
}

// The fp16 tail of one (sequence, head), lane = channel sl*32 + lane; adds into the
// warp's shared [G][128] channel sums.
template <int G>
__device__ __forceinline__ void pv_tail(const GemvArgs& a, long bh, int nb, int tl, float* sacc, int lane) {
  const long b = bh / a.kv_heads, h = bh % a.kv_heads;
  const uint16_t* tail = a.tail + (size_t)bh * 128 * 128;
  float acc[4][G];
#pragma unroll
  for (int sl = 0; sl < 4; ++sl)
#pragma unroll
    for (int hd = 0; hd < G; ++hd) acc[sl][hd] = 0.f;
  for (int t = 0; t < tl; ++t) {
    float vv[4];
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) vv[sl] = half_bits_to_float(tail[(size_t)t * 128 + sl * 32 + lane]);
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      const float pt = a.p[head_row(a, b, h, hd) * a.ld + (long)nb * 128 + t];
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = fmaf(pt, vv[sl], acc[sl][hd]);
    }
  }
#pragma unroll
  for (int sl = 0; sl < 4; ++sl)
#pragma unroll
    for (int hd = 0; hd < G; ++hd) sacc[hd * 128 + sl * 32 + lane] += acc[sl][hd];
}

// Zeroes a warp's [G][128] channel sums.
template <int G>
__device__ __forceinline__ void zero_sums(float* sacc, int lane) {
  float4* p = reinterpret_cast<float4*>(sacc);
#pragma unroll
  for (int i = lane; i < G * 32; i += 32) p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace

}  // namespace packkv
