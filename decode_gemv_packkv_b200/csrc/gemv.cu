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
//    partials, writes them to the workspace at every (sequence, head) boundary,
//    and the last warp to finish a (sequence, head) (atomic counter, no waiting)
//    adds the partials in warp order: deterministic, no second kernel.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "kernels.h"

namespace packkv {

namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kWarpSmemBudget = 27 * 1024;  // two CTAs of 4 warps per SM
constexpr uint32_t kMagicBits = 0x4B000000u;
constexpr float kMagic = 8388608.0f;

enum ItemKind : int { kKindRaw = 0, kKindPacked = 1, kKindInvalid = 2, kKindTail = 3 };

__device__ __forceinline__ float mag(uint32_t field_bits) {
  return __uint_as_float(field_bits | kMagicBits) - kMagic;
}

// Field position exponents of the in-register decode (value = field * 2^sig).
__host__ __device__ constexpr int sig4(int i) { return i <= 4 ? 4 * i : 4 * i - 12; }
__host__ __device__ constexpr int sig2(int i) { return i <= 10 ? 2 * i : 2 * i - 12; }
__host__ __device__ constexpr float pow2(int e) {
  return e >= 0 ? float(1u << e) : 1.0f / float(1u << (-e));
}

// 8 nibbles of a 4-bit slice word: v[i] = field_i * 2^sig4(i)
__device__ __forceinline__ void dec4(uint32_t w, float (&v)[8]) {
  const uint32_t h = w >> 12;
  v[0] = mag(w & 0xFu);
  v[1] = mag(w & 0xF0u);
  v[2] = mag(w & 0xF00u);
  v[3] = mag(w & 0xF000u);
  v[4] = mag(w & 0xF0000u);
  v[5] = mag(h & 0xF00u);
  v[6] = mag(h & 0xF000u);
  v[7] = mag(h & 0xF0000u);
}

// 16 two-bit fields of a 2-bit slice word: v[i] = field_i * 2^sig2(i)
__device__ __forceinline__ void dec2(uint32_t w, float (&v)[16]) {
  const uint32_t h = w >> 12;
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = (i <= 10) ? mag(w & (3u << (2 * i))) : mag(h & (3u << (2 * i - 12)));
}

// 3-bit raw unit, 16 tokens: 2-bit slice word w2 plus the 16 slice-1 bits at bits 0..15 of x.
// v[i] = (field2_i + 4*bit_i) * 2^sig2(i), merged with one exact FFMA.
__device__ __forceinline__ void dec3(uint32_t w2, uint32_t x, float (&v)[16]) {
  dec2(w2, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = fmaf(mag(x & (1u << i)), pow2(sig2(i) - i + 2), v[i]);
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
  static constexpr int kStageRec = 528 + kChunks * kPitch;     // >= every record of this width
  static constexpr int kStageBytes = kStageRec + (PV ? 512 * G : 0);
  static constexpr int kTableBytes = 512 * G;
  static constexpr int kStages0 = (kWarpSmemBudget - kTableBytes - 64) / kStageBytes;
  static constexpr int kStages = kStages0 > 4 ? 4 : (kStages0 < 2 ? 2 : kStages0);
  static constexpr int kWarpSmem = ((kStages * kStageBytes + kTableBytes + kStages * 16) + 127) / 128 * 128;
  // q' table: channel c = h*kChanPerChunk + cc stored at ((cc/4)*NH + h)*4 + cc%4
  static constexpr int kNH = 128 / kChanPerChunk;
};

template <int BITS, int G, bool PV>
__device__ __forceinline__ int table_index(int c) {
  using C = Cfg<BITS, G, PV>;
  const int h = c / C::kChanPerChunk, cc = c % C::kChanPerChunk;
  return ((cc >> 2) * C::kNH + h) * 4 + (cc & 3);
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

// Issue the copies of item x into stage s (whole warp participates).
template <int BITS, int G, bool PV>
__device__ __forceinline__ void issue_item(const GemvArgs& a, const WarpMem<BITS, G, PV>& m, long x, int s,
                                           int lane) {
  using C = Cfg<BITS, G, PV>;
  const long bh = x / a.items_per_bh;
  const int j = (int)(x % a.items_per_bh);
  int kind = kKindTail;
  uint64_t off16 = 0;
  uint32_t len16 = 0;
  if (j < a.n_blocks) {
    const uint2 e = *reinterpret_cast<const uint2*>(a.index + ((size_t)bh * a.max_blocks + j) * 2);
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
  if (kind == kKindRaw) {
    if (lane < C::kChunks)
      bulk_g2s(st + 528 + lane * C::kPitch, src + 528 + lane * C::kChunkBytes, C::kChunkBytes, m.bar(s));
    if (lane == 16) bulk_g2s(st, src, 528, m.bar(s));
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
// q·Kᵀ
// ----------------------------------------------------------------------------
template <int BITS, int G>
__device__ __forceinline__ void qk_raw(const unsigned char* st, const float* qp, const float (&cst)[G],
                                       float* srow0, long ld, float scale, int lane) {
  using C = Cfg<BITS, G, false>;
  if constexpr (BITS == 4) {
    const int h = lane & 1, k = (lane >> 1) & 3, g = lane >> 3;
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (2 * g + h) * C::kPitch) + k;
    float acc[G][8];
#pragma unroll
    for (int hd = 0; hd < G; ++hd)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[hd][i] = 0.f;
#pragma unroll 2
    for (int c4 = 0; c4 < 16; ++c4) {
      float4 qv[G];
#pragma unroll
      for (int hd = 0; hd < G; ++hd)
        qv[hd] = *reinterpret_cast<const float4*>(qp + hd * 128 + (c4 * C::kNH + h) * 4);
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) w[t] = wp[4 * (c4 * 4 + t)];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float v[8];
        dec4(w[t], v);
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          const float qq = t == 0 ? qv[hd].x : t == 1 ? qv[hd].y : t == 2 ? qv[hd].z : qv[hd].w;
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[hd][i] = fmaf(qq, v[i], acc[hd][i]);
        }
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[hd][i] += __shfl_xor_sync(0xffffffffu, acc[hd][i], 1);
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = acc[hd][i] * pow2(-sig4(i));
        const float hi = acc[hd][i + 4] * pow2(-sig4(i + 4));
        o[i] = scale * (cst[hd] + (h ? hi : lo));
      }
      float* dst = srow0 + hd * ld + 32 * g + 8 * k + 4 * h;
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    }
  } else {
    const int h = lane & 3, k = (lane >> 2) & 1, g = lane >> 3;
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (4 * g + h) * C::kPitch);
    float acc[G][16];
#pragma unroll
    for (int hd = 0; hd < G; ++hd)
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[hd][i] = 0.f;
#pragma unroll 1
    for (int c4 = 0; c4 < 8; ++c4) {
      float4 qv[G];
#pragma unroll
      for (int hd = 0; hd < G; ++hd)
        qv[hd] = *reinterpret_cast<const float4*>(qp + hd * 128 + (c4 * C::kNH + h) * 4);
      uint32_t w[4], x[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int cc = c4 * 4 + t;
        if constexpr (BITS == 2) {
          w[t] = wp[2 * cc + k];
        } else {
          w[t] = wp[3 * cc + k];
          x[t] = wp[3 * cc + 2] >> (16 * k);
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float v[16];
        if constexpr (BITS == 2)
          dec2(w[t], v);
        else
          dec3(w[t], x[t], v);
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          const float qq = t == 0 ? qv[hd].x : t == 1 ? qv[hd].y : t == 2 ? qv[hd].z : qv[hd].w;
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[hd][i] = fmaf(qq, v[i], acc[hd][i]);
        }
      }
    }
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        acc[hd][i] += __shfl_xor_sync(0xffffffffu, acc[hd][i], 1);
        acc[hd][i] += __shfl_xor_sync(0xffffffffu, acc[hd][i], 2);
      }
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = 0.f;
#pragma unroll
        for (int hh = 0; hh < 4; ++hh)
          if (h == hh) v = acc[hd][4 * hh + i] * pow2(-sig2(4 * hh + i));
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
__device__ __forceinline__ void qk_packed(const unsigned char* st, const float* qp, const float (&cst)[G],
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
        part = fmaf(qp[hd * 128 + table_index<BITS, G, false>(4 * lane + i)], (float)((m4 >> (8 * i)) & 15u), part);
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
          acc[hd] = fmaf(qp[hd * 128 + table_index<BITS, G, false>(4 * c4 + i)], u, acc[hd]);
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
  for (int s = 0; s < C::kStages && prod < hi; ++s, ++prod) issue_item<BITS, G, false>(a, m, prod, s, lane);

  const int q_heads = a.kv_heads * G;
  long cur_bh = -1;
  float qr[G][4];
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x) {
    const long bh = x / a.items_per_bh;
    const int j = (int)(x % a.items_per_bh);
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
      // per-block q' = q * scale_c (table) and the min term sum_c q_c * mn_c
      float* qp = m.table();
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      float cst[G];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        float part = qr[hd][0] * mn0.x;
        part = fmaf(qr[hd][1], mn0.y, part);
        part = fmaf(qr[hd][2], mn1.x, part);
        part = fmaf(qr[hd][3], mn1.y, part);
        cst[hd] = warp_sum(part);
        *reinterpret_cast<float4*>(qp + hd * 128 + table_index<BITS, G, false>(4 * lane)) =
            make_float4(qr[hd][0] * sc0.x, qr[hd][1] * sc0.y, qr[hd][2] * sc1.x, qr[hd][3] * sc1.y);
      }
      __syncwarp();
      float* sblk = srow0 + (long)j * 128;
      if (kind == kKindRaw)
        qk_raw<BITS, G>(st, qp, cst, sblk, a.ld, a.scale, lane);
      else
        qk_packed<BITS, G>(st, qp, cst, sblk, a.ld, a.scale, lane);
    }
    __syncwarp();
    if (prod < hi) {
      issue_item<BITS, G, false>(a, m, prod, s, lane);
      ++prod;
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
}

// ----------------------------------------------------------------------------
// p·V
// ----------------------------------------------------------------------------
// Accumulates one raw block into acc[slab][hd] (lane = channel slab*32 + lane).
template <int BITS, int G>
__device__ __forceinline__ void pv_raw(const unsigned char* st, const float* pp, float (&acc)[4][G], int lane) {
  using C = Cfg<BITS, G, true>;
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      float v[32];
      if constexpr (BITS == 4) {
        const uint4 u = *reinterpret_cast<const uint4*>(st + 528 + (2 * g + (sl >> 1)) * C::kPitch +
                                                        ((sl & 1) * 32 + lane) * 16);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float t[8];
          dec4(w[q], t);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[8 * q + i] = t[i];
        }
      } else if constexpr (BITS == 2) {
        const uint2 u = *reinterpret_cast<const uint2*>(st + 528 + (4 * g + sl) * C::kPitch + lane * 8);
        float t[16];
        dec2(u.x, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = t[i];
        dec2(u.y, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 + i] = t[i];
      } else {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(st + 528 + (4 * g + sl) * C::kPitch + lane * 12);
        const uint32_t w0 = wp[0], w1 = wp[1], w2 = wp[2];
        float t[16];
        dec3(w0, w2, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = t[i];
        dec3(w1, w2 >> 16, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 + i] = t[i];
      }
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4* p4 = reinterpret_cast<const float4*>(pp + hd * 128 + 32 * g);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 pv = p4[q];
          a0 = fmaf(pv.x, v[4 * q + 0], a0);
          a1 = fmaf(pv.y, v[4 * q + 1], a1);
          a0 = fmaf(pv.z, v[4 * q + 2], a0);
          a1 = fmaf(pv.w, v[4 * q + 3], a1);
        }
        acc[sl][hd] += a0 + a1;
      }
    }
  }
}

template <int BITS, int G>
__device__ __forceinline__ void pv_packed(const unsigned char* st, const float* pp, const float (&pg)[G][4],
                                          float (&acc)[4][G], int lane) {
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
        acc[sl][hd] += sum;
      }
    }
  }
}

// Writes this warp's partial sums for (b, h) and, if it is the last warp of
// that (b, h) to do so, reduces all partials in warp order into `out`.
template <int G>
__device__ __forceinline__ void pv_flush(const GemvArgs& a, long bh, int warp, float (&acc)[4][G], float (&mp)[G],
                                         int lane) {
  const long slot = warp + bh;
  float* part = a.partials + (size_t)slot * G * 128;
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    const float mn = warp_sum(mp[hd]);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) __stcg(part + hd * 128 + sl * 32 + lane, acc[sl][hd] + mn);
  }
  __threadfence();
  // warps that touch this (b, h): items [bh*I, (bh+1)*I) over ranges floor(w*N/W)
  const long N = a.n_items, Wn = a.n_warps, I = a.items_per_bh;
  auto warp_of = [&](long item) -> long { return (long)(((long long)(item + 1) * Wn + N - 1) / N) - 1; };
  const long w0 = warp_of(bh * I), w1 = warp_of((bh + 1) * I - 1);
  unsigned int prev = 0;
  if (lane == 0) prev = atomicAdd(a.counters + bh, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev == (unsigned int)(w1 - w0)) {
    __threadfence();
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
#pragma unroll 1
    for (int hd = 0; hd < G; ++hd) {
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        float sum = 0.f;
        for (long w = w0; w <= w1; ++w) sum += __ldcg(a.partials + (size_t)(w + bh) * G * 128 + hd * 128 + sl * 32 + lane);
        a.out[((size_t)b * a.kv_heads * G + h * G + hd) * 128 + sl * 32 + lane] = sum;
      }
    }
    if (lane == 0) a.counters[bh] = 0u;
  }
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    mp[hd] = 0.f;
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = 0.f;
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
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(m.bar(s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  long prod = lo;
  for (int s = 0; s < C::kStages && prod < hi; ++s, ++prod) issue_item<BITS, G, true>(a, m, prod, s, lane);

  float acc[4][G], mp[G];
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    mp[hd] = 0.f;
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = 0.f;
  }
  long cur_bh = lo / a.items_per_bh;
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x) {
    const long bh = x / a.items_per_bh;
    const int j = (int)(x % a.items_per_bh);
    if (bh != cur_bh) {
      pv_flush<G>(a, cur_bh, warp, acc, mp, lane);
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
          for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = fmaf(pt, vv[sl], acc[sl][hd]);
        }
      }
    } else if (kind == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
    } else {
      // p' = p * scale_r (with the field exponent folded in for raw blocks) and the min term
      float* pp = m.table();
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      const float mnr[4] = {mn0.x, mn0.y, mn1.x, mn1.y};
      const float scr[4] = {sc0.x, sc0.y, sc1.x, sc1.y};
      float pg[G][4];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 p4 = *reinterpret_cast<const float4*>(st + C::kStageRec + hd * 512 + 16 * lane);
        const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
        float o[4];
        float ps = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mp[hd] = fmaf(pr[i], mnr[i], mp[hd]);
          const float pprime = pr[i] * scr[i];
          ps += pprime;
          const int r = 4 * lane + i;  // storage slot
          float e;
          if constexpr (BITS == 4)
            e = pow2(-sig4(r & 7));
          else
            e = pow2(-sig2(r & 15));
          // (r & 7) / (r & 15) depend only on lane parity classes; the exponent is exact
          o[i] = kind == kKindRaw ? pprime * e : pprime;
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
    __syncwarp();
    if (prod < hi) {
      issue_item<BITS, G, true>(a, m, prod, s, lane);
      ++prod;
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
  pv_flush<G>(a, cur_bh, warp, acc, mp, lane);
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
  return cudaLaunchKernel(info.fn, dim3(grid), dim3(kWarpsPerCta * 32), args, info.smem, stream);
}

}  // namespace

int gemv_max_warps() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * 64;
}

size_t pv_workspace_bytes(int batch, int kv_heads, int group) {
  const size_t bh = (size_t)batch * kv_heads;
  const size_t counters = (bh * 4 + 255) / 256 * 256;
  return counters + ((size_t)gemv_max_warps() + bh) * group * 128 * sizeof(float);
}

cudaError_t launch_qk(GemvArgs a, cudaStream_t stream) { return launch<false>(a, stream); }
cudaError_t launch_pv(GemvArgs a, cudaStream_t stream) { return launch<true>(a, stream); }

}  // namespace packkv
