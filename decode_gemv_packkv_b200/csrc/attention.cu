// Fused decode attention over the packed cache (PackKV paper page, Figure 1: the
// scores, the softmax between them and the weighted sum of values that make up
// decode attention; Figure 2: the decompression folded into both products).
//
//   out[b,hq,c] = sum_i softmax_i(scale * q[b,hq]·k_hat[b,h,i]) * v_hat[b,h,i,c]
//
// over the packed blocks (storage order) and the fp16 tail.  One pass over both
// arenas: a warp owns a contiguous range of items (blocks, then the tail) of the
// flat (sequence, kv-head) list, as the q·Kᵀ / p·V kernels do.  Per item it
// stages the K record, then the V record in the same shared-memory stage (the V
// copy is issued as soon as q·Kᵀ has read the K record, the next K copy as soon
// as p·V has read the V record), computes the item's scores into shared memory with the
// q·Kᵀ decode paths, updates a running maximum and sum of exponentials per head
// (online softmax), and adds the probability-weighted values with the p·V decode
// paths.  At every (sequence, head) boundary it writes its sums, maximum and sum
// of exponentials per query head to its workspace slot; a second kernel,
// launched as a programmatic dependent, merges the slots of each (sequence,
// head) in warp order with the log-sum-exp rule: deterministic.  Neither the
// scores nor the probabilities ever reach global memory.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "decode.cuh"

namespace packkv {

namespace {

#ifndef PACKKV_ATTN_WARPS_PER_CTA
#define PACKKV_ATTN_WARPS_PER_CTA 4
#endif
constexpr int kAttnWarps = PACKKV_ATTN_WARPS_PER_CTA;
#ifndef PACKKV_ATTN_ONE_STAGE
// 1: an item's K and V records share one stage, loaded one after the other (half the
// shared memory per warp, twice the resident warps: measured faster than two stages)
#define PACKKV_ATTN_ONE_STAGE 1
#endif
constexpr bool kOneStage = PACKKV_ATTN_ONE_STAGE != 0;
constexpr int kAttnStages = kOneStage ? 1 : 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSlotFloats = 132;  // per (workspace slot, head): 128 sums, running max, sum of exp, pad
constexpr float kNegInf = -__builtin_huge_valf();

template <int BITS, int G>
struct AttnCfg {
  using C = Cfg<BITS, G, false>;
  static constexpr int kStageRec = C::kStageRec;  // one K or one V record
  static constexpr int kNT = C::kNT;
  static constexpr int kI8Tab = C::kI8Tab;
  static constexpr int kTableBytes = (kI8Tab + 15) / 16 * 16;
  static constexpr int kScoreBytes = 512 * G;  // [G][128] scores, then probabilities
  static constexpr int kSumBytes = 512 * G;    // [G][128] channel sums (compressed records and the tail)
  static constexpr int kFixed = kAttnStages * kStageRec + kTableBytes + kScoreBytes + kSumBytes;
  static constexpr int kWarpSmem = (kFixed + 32 + 127) / 128 * 128;
  static_assert(kStageRec % 16 == 0 && kFixed % 16 == 0, "stage alignment");
};

// Warp-private shared memory: [K stage][V stage][table][scores][sums][2 mbarriers][2 kinds].
template <int BITS, int G>
struct AttnMem {
  using A = AttnCfg<BITS, G>;
  unsigned char* base;
  __device__ unsigned char* stage(int s) const { return base + (kOneStage ? 0 : s) * A::kStageRec; }
  __device__ uint32_t* table() const { return reinterpret_cast<uint32_t*>(base + kAttnStages * A::kStageRec); }
  __device__ float* scores() const {
    return reinterpret_cast<float*>(base + kAttnStages * A::kStageRec + A::kTableBytes);
  }
  __device__ float* sums() const { return scores() + 128 * G; }
  __device__ uint64_t* bar(int s) const { return reinterpret_cast<uint64_t*>(base + A::kFixed) + s; }
  __device__ int* kind(int s) const { return reinterpret_cast<int*>(base + A::kFixed + 16) + s; }
};

// The K (v = false) or V (v = true) half of the arguments, in the form the shared
// staging and decode helpers take.
__device__ __forceinline__ GemvArgs tensor_view(const AttnArgs& a, bool v) {
  GemvArgs g{};
  g.arena = v ? a.v_arena : a.k_arena;
  g.index = v ? a.v_index : a.k_index;
  g.tail = v ? a.v_tail : a.k_tail;
  g.batch = a.batch;
  g.kv_heads = a.kv_heads;
  g.group = a.group;
  g.g_total = a.g_total;
  g.g_off = a.g_off;
  g.max_blocks = a.max_blocks;
  g.n_blocks = a.n_blocks;
  g.tail_len = a.tail_len;
  g.bits = a.bits;
  g.arena16 = a.arena16;
  g.ctrl = a.ctrl;
  g.n_items = a.n_items;
  g.items_per_bh = a.items_per_bh;
  g.n_warps = a.n_warps;
  g.block_table = a.block_table;
  g.ragged = a.ragged;
  return g;
}

// Scaled scores of the fp16 tail tokens of (sequence, head) bh into sc[head*128 + t].
template <int G>
__device__ __forceinline__ void tail_scores(const AttnArgs& a, long bh, int tl, const float (&qr)[G][4], float* sc,
                                            int lane) {
  const uint16_t* tail = a.k_tail + (size_t)bh * 128 * 128;
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
      for (int hd = 0; hd < G; ++hd) sc[hd * 128 + t0 + lane] = a.scale * mine[hd];
    }
  }
}

// Adds sum_t p[head][t] * v_tail[t][c] into the channel sums (lane = channel sl*32 + lane).
template <int G>
__device__ __forceinline__ void tail_values(const AttnArgs& a, long bh, int tl, const float* p, float* sacc,
                                            int lane) {
  const uint16_t* tail = a.v_tail + (size_t)bh * 128 * 128;
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
      const float pt = p[hd * 128 + t];
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) acc[sl][hd] = fmaf(pt, vv[sl], acc[sl][hd]);
    }
  }
#pragma unroll
  for (int sl = 0; sl < 4; ++sl)
#pragma unroll
    for (int hd = 0; hd < G; ++hd) sacc[hd * 128 + sl * 32 + lane] += acc[sl][hd];
}

// Writes this warp's state for (b, h) to its slot (warp + bh) and clears it: per query
// head the 128 value sums (tensor-core accumulators, channel sums and the min term
// together), the running maximum and the running sum of exponentials.
template <int G>
__device__ __forceinline__ void attn_flush(const AttnArgs& a, long bh, int warp, float* sacc,
                                           float (&acc_lo)[I8Layout<G>::kNH][8],
                                           float (&acc_hi)[I8Layout<G>::kNH][8], float (&mp)[G], float (&mrun)[G],
                                           float (&lrun)[G], int lane) {
  using L = I8Layout<G>;
  const int g = lane >> 2, t = lane & 3;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < L::kNH; ++j) {
    const int head = L::head(j, t);
#pragma unroll
    for (int T = 0; T < 8; ++T) {
      if (L::owns(j, t)) {
        sacc[head * 128 + 16 * T + g] += acc_lo[j][T];
        sacc[head * 128 + 16 * T + g + 8] += acc_hi[j][T];
      }
      acc_lo[j][T] = 0.f;
      acc_hi[j][T] = 0.f;
    }
  }
  __syncwarp();
  float* part = a.partials + (size_t)(warp + bh) * G * kSlotFloats;
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    const float mn = warp_sum(mp[hd]);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int c = sl * 32 + lane;
      __stcg(part + hd * kSlotFloats + c, sacc[hd * 128 + c] + mn);
    }
    if (lane == 0) {
      __stcg(part + hd * kSlotFloats + 128, mrun[hd]);
      __stcg(part + hd * kSlotFloats + 129, lrun[hd]);
    }
    mp[hd] = 0.f;
    mrun[hd] = kNegInf;
    lrun[hd] = 0.f;
  }
  __syncwarp();
  zero_sums<G>(sacc, lane);
  __syncwarp();
}

// Resident CTAs per SM the register budget is sized for: shared memory admits five
// 4-warp CTAs of the 2- and 4-bit single-head kernels, which then need <= 102 registers.
constexpr int attn_min_ctas(int bits, int g) { return kAttnWarps == 4 && g == 1 && bits != 3 ? 5 : 0; }

template <int BITS, int G, class Plan>
__global__ void __launch_bounds__(kAttnWarps * 32, attn_min_ctas(BITS, G))
    attn_kernel(const AttnArgs a, const __grid_constant__ Plan plan) {
  using A = AttnCfg<BITS, G>;
  using C = Cfg<BITS, G, false>;
  constexpr int NT = A::kNT;
  constexpr int NH = C::kNH;
  extern __shared__ __align__(128) unsigned char smem[];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kAttnWarps + (threadIdx.x >> 5);
  if (warp >= a.n_warps) return;
  const AttnMem<BITS, G> m{smem + (threadIdx.x >> 5) * A::kWarpSmem};
  const GemvArgs ka = tensor_view(a, false), va = tensor_view(a, true);
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    mbar_init(m.bar(0), 1);
    mbar_init(m.bar(1), 1);
    fence_mbar_init();
  }
  __syncwarp();
  Cursor cc = cursor_at(a, plan, lo);
  EntryWindow wk, wv;
  wk.load(ka, plan, lo, hi, lane);
  wv.load(va, plan, lo, hi, lane);
  issue_item<BITS, G, false>(ka, m, cc, wk.get(lo), 0, lane);
  if (!kOneStage) issue_item<BITS, G, false>(va, m, cc, wv.get(lo), 1, lane);

  float qr[G][4];
  float mrun[G], lrun[G], mp[G];
  float acc_lo[NH][8], acc_hi[NH][8];
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    mrun[hd] = kNegInf;
    lrun[hd] = 0.f;
    mp[hd] = 0.f;
  }
#pragma unroll
  for (int jn = 0; jn < NH; ++jn)
#pragma unroll
    for (int T = 0; T < 8; ++T) acc_lo[jn][T] = acc_hi[jn][T] = 0.f;
  float* sacc = m.sums();
  float* sc = m.scores();
  zero_sums<G>(sacc, lane);
  __syncwarp();
  long cur_bh = -1;
  uint32_t phases = 0;
  const int g = lane >> 2, t = lane & 3;
  for (long x = lo; x < hi; ++x) {
    const long bh = cc.bh;
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    if (bh != cur_bh) {
      if (cur_bh >= 0) attn_flush<G>(a, cur_bh, warp, sacc, acc_lo, acc_hi, mp, mrun, lrun, lane);
      cur_bh = bh;
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const uint2 hv = *reinterpret_cast<const uint2*>(a.q + head_row(a, b, h, hd) * 128 + 4 * lane);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
        qr[hd][0] = f0.x;
        qr[hd][1] = f0.y;
        qr[hd][2] = f1.x;
        qr[hd][3] = f1.y;
      }
    }
    Cursor nc = cc;
    cursor_next(a, plan, nc);

    // ---- K: scaled scores of this item's tokens into sc[head][slot] ----------
    bool ok = mbar_wait_bounded(m.bar(0), phases & 1u, a.ctrl);
    phases ^= 1u;
    if (!ok) {  // the copy never landed (status set): wait, bounded, for the V copy, then stop
      if (!kOneStage) mbar_wait_bounded(m.bar(1), (phases >> 1) & 1u, a.ctrl);
      return;
    }
    const int kind_len_k = *m.kind(0);
    const int kind_k = kind_len_k & 0xFF;
    int n_tok = 128;
    bool skip = false;
    if (kind_k == kKindTail) {
      n_tok = cc.tl;
      tail_scores<G>(a, bh, cc.tl, qr, sc, lane);
    } else if (kind_k == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
      skip = true;
    } else {
      unsigned char* st = m.stage(0);
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      float cst[G], qv[G][4];
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
      uint32_t* tab = m.table();
      float invf[G];
      build_i8tab<G, NT>(tab, qv, invf, lane);
      __syncwarp();
      if (kind_k == kKindRaw) {
        qk_i8<BITS, G>(st, tab, cst, invf, sc, 128, a.scale, lane);
      } else if (!qk_packed_tc<BITS, G>(st, (uint32_t)(kind_len_k >> 8) * 16u, tab, qv, cst, invf, sc, 128, a.scale,
                                         lane)) {
        if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
        skip = true;
      }
    }
    __syncwarp();
    if (kOneStage) {  // the stage is free: this item's V record
      if (x - wv.base >= 32) wv.load(va, plan, x, hi, lane);
      issue_item<BITS, G, false>(va, m, cc, wv.get(x), 1, lane);
    } else if (x + 1 < hi) {  // the K stage is free: the next item's K record
      if (x + 1 - wk.base >= 32) wk.load(ka, plan, x + 1, hi, lane);
      issue_item<BITS, G, false>(ka, m, nc, wk.get(x + 1), 0, lane);
    }

    // ---- online softmax: running max and sum of exp per head, p of this lane's slots
    float pr[G][4];
#pragma unroll
    for (int hd = 0; hd < G; ++hd) {
      float sv[4];
      float bm = kNegInf;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * lane + i;
        sv[i] = (!skip && r < n_tok) ? sc[hd * 128 + r] : kNegInf;
        bm = fmaxf(bm, sv[i]);
      }
      bm = warp_max(bm);
      const float m_new = fmaxf(mrun[hd], bm);
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        pr[hd][i] = sv[i] == kNegInf ? 0.f : exp2f((sv[i] - m_new) * kLog2e);
        ps += pr[hd][i];
      }
      ps = warp_sum(ps);
      if (m_new > mrun[hd]) {  // warp-uniform: rescale what was summed under the old max
        const float alpha = mrun[hd] == kNegInf ? 0.f : exp2f((mrun[hd] - m_new) * kLog2e);
        lrun[hd] *= alpha;
        mp[hd] *= alpha;
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) sacc[hd * 128 + sl * 32 + lane] *= alpha;
#pragma unroll
        for (int jn = 0; jn < NH; ++jn) {
          if (I8Layout<G>::head(jn, t) == hd) {
#pragma unroll
            for (int T = 0; T < 8; ++T) {
              acc_lo[jn][T] *= alpha;
              acc_hi[jn][T] *= alpha;
            }
          }
        }
        mrun[hd] = m_new;
      }
      lrun[hd] += ps;
    }

    // ---- V: add the probability-weighted values -------------------------------
    ok = mbar_wait_bounded(m.bar(1), (phases >> 1) & 1u, a.ctrl);
    phases ^= 2u;
    if (!ok) {
      if (!kOneStage && x + 1 < hi) mbar_wait_bounded(m.bar(0), phases & 1u, a.ctrl);
      return;
    }
    const int kind_len_v = *m.kind(1);
    const int kind_v = kind_len_v & 0xFF;
    if (kind_v == kKindTail) {
#pragma unroll
      for (int hd = 0; hd < G; ++hd)
        *reinterpret_cast<float4*>(sc + hd * 128 + 4 * lane) = make_float4(pr[hd][0], pr[hd][1], pr[hd][2], pr[hd][3]);
      __syncwarp();
      tail_values<G>(a, bh, cc.tl, sc, sacc, lane);
    } else if (kind_v == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
    } else if (!skip) {
      unsigned char* st = m.stage(1);
      const uint2 mnv = *reinterpret_cast<const uint2*>(st + kParamOffset + 8 * lane);
      const uint2 scv = *reinterpret_cast<const uint2*>(st + kParamOffset + 256 + 8 * lane);
      const float2 mn0 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.x));
      const float2 mn1 = __half22float2(*reinterpret_cast<const __half2*>(&mnv.y));
      const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&scv.x));
      const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&scv.y));
      const float mnr[4] = {mn0.x, mn0.y, mn1.x, mn1.y};
      const float scr[4] = {sc0.x, sc0.y, sc1.x, sc1.y};
      float pv4[G][4];
      float mpr[G];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        mpr[hd] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mpr[hd] = fmaf(pr[hd][i], mnr[i], mpr[hd]);
          pv4[hd][i] = pr[hd][i] * scr[i];
        }
      }
      uint32_t* tab = m.table();
      float invf[G];
      build_i8tab<G, NT>(tab, pv4, invf, lane);
      __syncwarp();
      bool ok = true;
      if (kind_v == kKindRaw)
        pv_i8<BITS, G>(st, tab, invf, acc_lo, acc_hi, lane);
      else
        ok = pv_packed_nat<BITS, G>(st, (uint32_t)(kind_len_v >> 8) * 16u, tab, invf, sacc, lane);
      if (ok) {
#pragma unroll
        for (int hd = 0; hd < G; ++hd) mp[hd] += mpr[hd];
      } else if (lane == 0) {
        set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
      }
    }
    __syncwarp();
    if (x + 1 < hi) {
      if (kOneStage) {  // the stage is free: the next item's K record
        if (x + 1 - wk.base >= 32) wk.load(ka, plan, x + 1, hi, lane);
        issue_item<BITS, G, false>(ka, m, nc, wk.get(x + 1), 0, lane);
      } else {  // the V stage is free: the next item's V record
        if (x + 1 - wv.base >= 32) wv.load(va, plan, x + 1, hi, lane);
        issue_item<BITS, G, false>(va, m, nc, wv.get(x + 1), 1, lane);
      }
    }
    cc = nc;
  }
  (void)g;
  if (cur_bh >= 0) attn_flush<G>(a, cur_bh, warp, sacc, acc_lo, acc_hi, mp, mrun, lrun, lane);
}

// Warp whose item range holds `item` (ranges are [floor(w*N/W), floor((w+1)*N/W)), W <= N).
__device__ __forceinline__ long attn_warp_of_item(long item, long n_items, long n_warps) {
  return (long)(((long long)(item + 1) * n_warps + n_items - 1) / n_items) - 1;
}

// Second pass: for each output row (b, h, head), the slots of the warps that touched
// (b, h) are merged with the log-sum-exp rule, M = max m_w, L = sum l_w e^(m_w - M),
// out_c = sum S_w,c e^(m_w - M) / L, adding in a fixed order (deterministic).  One CTA
// per row: warp i of 32 takes slots w0+i, w0+i+32, ... (four loop iterations
// unrolled, so their loads overlap); warp 0 adds the 32 warp results in order.  A row
// whose every record was invalid gets NaN.
constexpr int kMergeWarps = 32;

template <int G, class Plan>
__global__ void __launch_bounds__(kMergeWarps * 32)
    attn_merge_kernel(const AttnArgs a, const __grid_constant__ Plan plan) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float4 wsum[kMergeWarps][32];
  __shared__ float wl[kMergeWarps];
  __shared__ float wmax[kMergeWarps];
  const long bh = blockIdx.x / G;  // block: (b*kv_heads + h)*G + head
  const int hd = (int)(blockIdx.x % G);
  const long row = (long)(head_row(a, bh / a.kv_heads, bh % a.kv_heads, hd));  // row of out
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long first = 0, n = 0;
  row_items(a, plan, bh, &first, &n);
  if (n == 0) {  // a sequence without tokens (ragged batches): its output is zero
    if (warp == 0) reinterpret_cast<float4*>(a.out + row * 128)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const long w0 = attn_warp_of_item(first, a.n_items, a.n_warps) + bh;
  const long w1 = attn_warp_of_item(first + n - 1, a.n_items, a.n_warps) + bh;
  const float* base = a.partials + hd * kSlotFloats;
  const size_t stride = (size_t)G * kSlotFloats;
  // the overall maximum
  float mx = kNegInf;
  for (long w = w0 + threadIdx.x; w <= w1; w += kMergeWarps * 32) mx = fmaxf(mx, __ldcg(base + w * stride + 128));
  mx = warp_max(mx);
  if (lane == 0) wmax[warp] = mx;
  __syncthreads();
  float M = wmax[0];
#pragma unroll
  for (int i = 1; i < kMergeWarps; ++i) M = fmaxf(M, wmax[i]);
  // scaled sums
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  float l = 0.f;
#pragma unroll 4
  for (long w = w0 + warp; w <= w1; w += kMergeWarps) {
    const float* p = base + w * stride;
    const float mw = __ldcg(p + 128);
    const float e = (mw == kNegInf) ? 0.f : exp2f((mw - M) * kLog2e);
    const float4 x = __ldcg(reinterpret_cast<const float4*>(p) + lane);
    s.x = fmaf(x.x, e, s.x);
    s.y = fmaf(x.y, e, s.y);
    s.z = fmaf(x.z, e, s.z);
    s.w = fmaf(x.w, e, s.w);
    l = fmaf(__ldcg(p + 129), e, l);
  }
  wsum[warp][lane] = s;
  if (lane == 0) wl[warp] = l;
  __syncthreads();
  if (warp == 0) {
    float4 r = wsum[0][lane];
    float L = wl[0];
#pragma unroll
    for (int i = 1; i < kMergeWarps; ++i) {
      const float4 x = wsum[i][lane];
      r.x += x.x;
      r.y += x.y;
      r.z += x.z;
      r.w += x.w;
      L += wl[i];
    }
    const float inv = L > 0.f ? 1.f / L : __int_as_float(0x7fc00000);
    reinterpret_cast<float4*>(a.out + row * 128)[lane] = make_float4(r.x * inv, r.y * inv, r.z * inv, r.w * inv);
  }
}

struct AttnKernel {
  const void* fn;
  int smem;
};

template <int BITS, int G, class Plan>
AttnKernel attn_info() {
  return {reinterpret_cast<const void*>(&attn_kernel<BITS, G, Plan>), kAttnWarps * AttnCfg<BITS, G>::kWarpSmem};
}

template <class Plan>
bool attn_select(int bits, int group, AttnKernel* out) {
#define PACKKV_ACASE(B, GG)            \
  if (bits == B && group == GG) {      \
    *out = attn_info<B, GG, Plan>();   \
    return true;                       \
  }
  PACKKV_ACASE(4, 1) PACKKV_ACASE(4, 2) PACKKV_ACASE(4, 4) PACKKV_ACASE(4, 8)
  PACKKV_ACASE(3, 1) PACKKV_ACASE(3, 2) PACKKV_ACASE(3, 4) PACKKV_ACASE(3, 8)
  PACKKV_ACASE(2, 1) PACKKV_ACASE(2, 2) PACKKV_ACASE(2, 4) PACKKV_ACASE(2, 8)
#undef PACKKV_ACASE
  return false;
}

// Resident warps of the kernel on the current device (configures the smem limit once).
cudaError_t attn_resident_warps(const AttnKernel& k, int* warps) {
  static std::mutex mu;
  static std::unordered_map<long long, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const long long key = (long long)(reinterpret_cast<uintptr_t>(k.fn)) * 64 + dev;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *warps = it->second;
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0, sms = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.fn, kAttnWarps * 32, k.smem);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int w = sms * per_sm * kAttnWarps;
  cache[key] = w;
  *warps = w;
  return cudaSuccess;
}

int attn_max_warps() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * 64;
}

}  // namespace

size_t attention_workspace_bytes(int batch, int kv_heads, int group) {
  const size_t bh = (size_t)batch * kv_heads;
  return ((size_t)attn_max_warps() + bh) * group * kSlotFloats * sizeof(float);
}

template <int G, class Plan>
const void* merge_fn() {
  return reinterpret_cast<const void*>(&attn_merge_kernel<G, Plan>);
}

template <class Plan>
cudaError_t launch_attention_t(AttnArgs a, const Plan* plan, cudaStream_t stream) {
  AttnKernel k{};
  if (!attn_select<Plan>(a.bits, a.group, &k)) return cudaErrorInvalidValue;
  int w = 0;
  cudaError_t e = attn_resident_warps(k, &w);
  if (e != cudaSuccess) return e;
  if (w > attn_max_warps()) w = attn_max_warps();
  a.n_warps = (int)(a.n_items < w ? a.n_items : w);
  if (a.n_warps < 1) a.n_warps = 1;
  const unsigned grid = (unsigned)((a.n_warps + kAttnWarps - 1) / kAttnWarps);
  void* args[] = {&a, const_cast<Plan*>(plan)};
  if (a.n_items > 0) {
    e = cudaLaunchKernel(k.fn, dim3(grid), dim3(kAttnWarps * 32), args, k.smem, stream);
    if (e != cudaSuccess) return e;
  }
  const void* merge = a.group == 1 ? merge_fn<1, Plan>() : a.group == 2 ? merge_fn<2, Plan>()
                    : a.group == 4 ? merge_fn<4, Plan>() : merge_fn<8, Plan>();
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)((long)a.batch * a.kv_heads * a.group));
  cfg.blockDim = dim3(kMergeWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.n_items > 0 ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, merge, args);
}

cudaError_t launch_attention(AttnArgs a, const RaggedPlan* plan, cudaStream_t stream) {
  static const NoPlan none{};
  return plan ? launch_attention_t<RaggedPlan>(a, plan, stream) : launch_attention_t<NoPlan>(a, &none, stream);
}

}  // namespace packkv
