// Device building blocks of the fused decode products over the packed cache:
// record staging (bulk copies into warp-private shared-memory stages, bounded
// mbarrier waits), the 8-bit integer tensor-core decode of raw records (2, 3 and
// 4-bit), and the CUDA-core decode of compressed records (packed-cache format v1, sections 3-4).  Included by the q·Kᵀ / p·V kernels and by the fused
// attention kernel.
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

template <int BITS, int G, bool PV>
struct Cfg {
  static constexpr int kRecBytes = raw_record_bytes(BITS);
  static constexpr int kStageRec = kRecBytes;                  // >= every record, staged in one piece
  static constexpr int kStageBytes = kStageRec;
  // int8 tensor-core B table: columns n = 4*head + digit (digit 3 = 0), NT n-tiles of 8
  static constexpr int kNT = I8Layout<G>::kNT;
  static constexpr int kNH = I8Layout<G>::kNH;
  static constexpr int kI8Tab = 4 * (64 * kNT + 8) * 4;
  // CUDA-core tables: q' [G][128] (q·Kᵀ); p'' [G][128] + group sums of p' [G][4] (p·V)
  static constexpr int kCoreTab = PV ? 512 * G + 16 * G : 512 * G;
  static constexpr int kTableBytes = ((kCoreTab > kI8Tab ? kCoreTab : kI8Tab) + 15) / 16 * 16;
  static constexpr int kSumBytes = PV ? 512 * G : 0;          // p·V: [G][128] channel sums
  static constexpr int kFixed = kTableBytes + kSumBytes;
  static constexpr int kStages0 = (kWarpSmemBudget - kFixed - 64) / kStageBytes;
  // p·V keeps the p of its in-flight record in registers, one record deep: one stage
  static constexpr int kStages = PV ? 1 : (kStages0 > 4 ? 4 : (kStages0 < 1 ? 1 : kStages0));
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

// Index entries {offset16, length16} of 32 consecutive items of a warp's range, one
// per lane ({0, 0} for a tail item or past the range), loaded with one coalesced
// load; any lane reads the entry of any item of the window by shuffle.
struct EntryWindow {
  long base;  // first item of the window
  uint2 ent;  // entry of item base + lane
  __device__ void load(const GemvArgs& a, long first, long hi, int lane) {
    base = first;
    ent = make_uint2(0u, 0u);
    const long item = first + lane;
    if (item < hi) {
      const long bh = item / a.items_per_bh;
      const int j = (int)(item % a.items_per_bh);
      if (j < a.n_blocks) ent = *reinterpret_cast<const uint2*>(a.index + ((size_t)bh * a.max_blocks + j) * 2);
    }
  }
  // Whole warp; base <= item < base + 32.
  __device__ uint2 get(long item) const {
    const int src = (int)(item - base);
    return make_uint2(__shfl_sync(0xffffffffu, ent.x, src), __shfl_sync(0xffffffffu, ent.y, src));
  }
};

// Issue the copies of item (bh, j) with index entry e into stage s of m (whole warp
// participates); m provides stage(s), bar(s) and kind(s).
template <int BITS, int G, bool PV, class Mem>
__device__ __forceinline__ void issue_item(const GemvArgs& a, const Mem& m, Cursor c, uint2 e, int s, int lane) {
  using C = Cfg<BITS, G, PV>;
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
// q·Kᵀ on the CUDA cores (compressed records)
// ----------------------------------------------------------------------------
// Exact float of an unsigned integer u < 2^23: u in the mantissa of 2^23, minus 2^23
// (two full-rate instructions instead of an integer-to-float conversion).
__device__ __forceinline__ float small_u2f(uint32_t u) { return __uint_as_float(u | 0x4B000000u) - 8388608.f; }

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

// One compressed K record, lane = token within each pack group.
template <int G>
__device__ __forceinline__ void qk_packed(const unsigned char* st, const float* qp, const float (&cst)[G],
                                          float* sblk, long ld, float scale, int lane) {
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
      const float4 q4 = *reinterpret_cast<const float4*>(qp + hd * 128 + 4 * lane);
      float part = q4.x * small_u2f(m4 & 15u);
      part = fmaf(q4.y, small_u2f((m4 >> 8) & 15u), part);
      part = fmaf(q4.z, small_u2f((m4 >> 16) & 15u), part);
      part = fmaf(q4.w, small_u2f((m4 >> 24) & 15u), part);
      bsum[hd] = warp_sum(part);
    }
    float acc[G];
#pragma unroll
    for (int hd = 0; hd < G; ++hd) acc[hd] = 0.f;
    int s = gws[g];
#pragma unroll 1
    for (int c4 = 0; c4 < 32; ++c4) {
      const uint32_t mm = *reinterpret_cast<const uint32_t*>(meta + g * 128 + 4 * c4);
      float q4[G][4];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 v = *reinterpret_cast<const float4*>(qp + hd * 128 + 4 * c4);
        q4[hd][0] = v.x;
        q4[hd][1] = v.y;
        q4[hd][2] = v.z;
        q4[hd][3] = v.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = (mm >> (8 * i + 4)) & 15u;
        const float u = small_u2f(unit_field(W, s, w, lane));
        s += w;
#pragma unroll
        for (int hd = 0; hd < G; ++hd) acc[hd] = fmaf(q4[hd][i], u, acc[hd]);
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) sblk[hd * ld + 32 * g + lane] = scale * (cst[hd] + bsum[hd] + acc[hd]);
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

// ----------------------------------------------------------------------------
// p·V on the CUDA cores (compressed records)
// ----------------------------------------------------------------------------
// One compressed V record, lane = channel sl*32 + lane; adds into the warp's shared
// [G][128] channel sums.  pg[hd*4 + g] = sum of p' over pack group g.
template <int G>
__device__ __forceinline__ void pv_packed(const unsigned char* st, const float* pp, const float* pg, float* sacc,
                                          int lane) {
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
      // this lane's unit (group g, channel c), eight tokens at a time: their offsets,
      // then p' * offset for a block of HB heads (one head at a time from G = 4 on, which
      // decodes the unit again per head but keeps the registers of the wider kernels)
      constexpr int HB = G >= 4 ? 1 : G;
      const int bit_word = start + ((w & 2) ? 2 : 0);  // the 1-bit slice follows the 2-bit one
      const uint32_t bit_hi = (w & 2) ? 2u : 0u;       // and is bit 2 of a width-3 unit
#pragma unroll 1
      for (int h0 = 0; h0 < G; h0 += HB) {
        float sum[HB];
#pragma unroll
        for (int h = 0; h < HB; ++h) sum[h] = (float)base * pg[(h0 + h) * 4 + g];
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // tokens 8k .. 8k+7
          float u[8];
          if (w == 4) {
            const uint32_t word = W[start + k];
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = small_u2f((word >> (4 * i)) & 15u);
          } else {
            uint32_t two = 0u, one = 0u;
            if (w & 2) two = W[start + (k >> 1)] >> (16 * (k & 1));
            if (w & 1) one = W[bit_word] >> (8 * k);
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = small_u2f(((two >> (2 * i)) & 3u) | (((one >> i) & 1u) << bit_hi));
          }
#pragma unroll
          for (int h = 0; h < HB; ++h) {
            const float4* pr4 = reinterpret_cast<const float4*>(pp + (h0 + h) * 128 + 32 * g + 8 * k);
            const float4 pa = pr4[0], pb = pr4[1];
            float t = sum[h];
            t = fmaf(pa.x, u[0], t);
            t = fmaf(pa.y, u[1], t);
            t = fmaf(pa.z, u[2], t);
            t = fmaf(pa.w, u[3], t);
            t = fmaf(pb.x, u[4], t);
            t = fmaf(pb.y, u[5], t);
            t = fmaf(pb.z, u[6], t);
            t = fmaf(pb.w, u[7], t);
            sum[h] = t;
          }
        }
#pragma unroll
        for (int h = 0; h < HB; ++h) sacc[(h0 + h) * 128 + c] += sum[h];
      }
    }
  }
}

// The fp16 tail of one (sequence, head), lane = channel sl*32 + lane; adds into the
// warp's shared [G][128] channel sums.
template <int G>
__device__ __forceinline__ void pv_tail(const GemvArgs& a, long bh, float* sacc, int lane) {
  const long b = bh / a.kv_heads, h = bh % a.kv_heads;
  const uint16_t* tail = a.tail + (size_t)bh * 128 * 128;
  float acc[4][G];
#pragma unroll
  for (int sl = 0; sl < 4; ++sl)
#pragma unroll
    for (int hd = 0; hd < G; ++hd) acc[sl][hd] = 0.f;
  for (int t = 0; t < a.tail_len; ++t) {
    float vv[4];
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) vv[sl] = half_bits_to_float(tail[(size_t)t * 128 + sl * 32 + lane]);
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      const float pt = a.p[((size_t)b * a.kv_heads * G + h * G + hd) * a.ld + (long)a.n_blocks * 128 + t];
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
