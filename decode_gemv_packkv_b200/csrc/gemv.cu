// Fused decompression + matrix-vector products over the packed cache
// (PackKV paper page, Figure 2: the decompression is folded into the
// matrix-vector multiplication; TL;DR: no decompressed data is written back;
// Figure 1: the two products of decode attention).
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
//    multicast).
//  * Dequantization is folded out of the inner loop: k_hat = mn_c + s_c*code
//    gives score = scale*(sum_c q_c mn_c + sum_c (q_c s_c) code); v_hat =
//    mn_r + s_r*code gives out_c = sum_r p_r mn_r + sum_r (p_r s_r) code.
//  * Raw records (2, 3 and 4 bits; the common case) hold their codes in the
//    fragment order of an 8-bit integer tensor-core operand: one AND per 32-bit
//    word yields a whole A register of four codes (times a known power of two;
//    3-bit records as a 2-bit plane and a 1-bit plane), and mma.sync m16n8k32
//    (u8 x s8 -> s32, exact) multiplies them by q' or p' written as three
//    base-128 digits of q'*f (f = 127 / max|q'| per record and head; about 22
//    significant bits, the digits in three B columns).
//  * Compressed (frame-of-reference) records also run on the int8 tensor cores
//    (decode.cuh, "Compressed records"): for q·Kᵀ the units of each pack group are
//    sorted by width so that every run of 16 units is decoded with one instruction
//    sequence; for p·V every lane decodes its units in natural channel order with the
//    same instructions whatever their widths.
//  * p·V: a warp sums its item range into per-channel fp32 partials and writes
//    them to the workspace at every (sequence, head) boundary (split-K over the
//    sequence); a second-pass kernel, launched as a programmatic dependent so
//    its launch overlaps the first, adds the partials of each (sequence, head)
//    in warp order: deterministic.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "decode.cuh"

namespace packkv {

namespace {

// Resident CTAs of 4 warps per SM that the register budget is sized for (0: the
// compiler's choice).  Shared memory admits 4-5 of them for the 2- and 4-bit
// kernels; without the hint the compiler may settle below 102 registers with spills.
// 4-bit, 8 heads: three CTAs per SM (168 registers) beat two (measured on 16 query rows
// per kv head: q·Kᵀ 60.9 against 66.0 us per call); at 2 and 3 bits that cap spills.
constexpr int qk_min_ctas(int bits, int g) {
  return kWarpsPerCta != 4 ? 0
         : g == 1 ? 5
         : g == 4 ? (bits == 2 ? 4 : bits == 4 ? 5 : 0)
                  : (g == 8 && bits == 4 ? 3 : 0);
}
constexpr int pv_min_ctas(int bits, int g) {
  return kWarpsPerCta != 4 ? 0 : g == 1 ? 5 : g == 4 ? (bits == 3 ? 0 : 4) : (g == 8 && bits == 4 ? 3 : 0);
}

template <int BITS, int G, class Plan>
__global__ void __launch_bounds__(kWarpsPerCta * 32, qk_min_ctas(BITS, G))
    qk_kernel(const GemvArgs a, const __grid_constant__ Plan plan) {
  using C = Cfg<BITS, G, false>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (warp >= a.n_warps) return;
  const WarpMem<BITS, G, false> m{smem + (threadIdx.x >> 5) * C::kWarpSmem};
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(m.bar(s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  long prod = lo;
  Cursor pc = cursor_at(a, plan, lo);
  Cursor cc = pc;
  EntryWindow win;
  win.load(a, plan, lo, hi, lane);
  for (int s = 0; s < C::kStages && prod < hi; ++s, ++prod, cursor_next(a, plan, pc))
    issue_item<BITS, G, false>(a, m, pc, win.get(prod), s, lane);

  long cur_bh = -1;
  float qr[G][4];
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x, cursor_next(a, plan, cc)) {
    const long bh = cc.bh;
    const int j = cc.j;
    const long b = bh / a.kv_heads, h = bh % a.kv_heads;
    float* srow0 = a.scores + head_row(a, b, h, 0) * a.ld;
    if (bh != cur_bh) {
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
    const bool ok = mbar_wait_bounded(m.bar(s), (phases >> s) & 1u, a.ctrl);
    phases ^= 1u << s;
    if (!ok) {  // the copy never landed: stop this warp (status already set)
      drain_stages<BITS, G, false>(m, phases, s, x, prod, a.ctrl);
      return;
    }
    const int kind_len = *m.kind(s);
    const int kind = kind_len & 0xFF;
    unsigned char* st = m.stage(s);
    if (kind == kKindTail) {
      qk_tail<G>(a, bh, cc.nb, cc.tl, qr, srow0, lane);
    } else if (kind == kKindInvalid) {
      if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
#pragma unroll
      for (int hd = 0; hd < G; ++hd)
        for (int i = lane; i < 128; i += 32) srow0[hd * a.ld + (long)j * 128 + i] = __int_as_float(0x7fc00000);
    } else {
      // per record: the min term sum_c q_c * mn_c, then q' = q * scale_c as the int8
      // tensor-core B table (raw and compressed records alike)
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
      uint32_t* tab = m.table();
      float invf[G];
      build_i8tab<G, C::kNT>(tab, qv, invf, lane);
      __syncwarp();
      if (kind == kKindRaw) {
        qk_i8<BITS, G>(st, tab, cst, invf, sblk, a.ld, a.scale, lane);
      } else if (!qk_packed_tc<BITS, G>(st, (uint32_t)(kind_len >> 8) * 16u, tab, qv, cst, invf, sblk, a.ld,
                                         a.scale, lane)) {
        if (lane == 0) set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
#pragma unroll
        for (int hd = 0; hd < G; ++hd)
          for (int i = lane; i < 128; i += 32) sblk[hd * a.ld + i] = __int_as_float(0x7fc00000);
      }
    }
    __syncwarp();
    if (prod < hi) {
      if (prod - win.base >= 32) win.load(a, plan, prod, hi, lane);
      issue_item<BITS, G, false>(a, m, pc, win.get(prod), s, lane);
      ++prod;
      cursor_next(a, plan, pc);
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
}

// Writes this warp's partial sums for (b, h) to its slot (warp + bh) and clears them:
// the tensor-core accumulators (even-t thread (g, t) holds channels 16T+g and 16T+g+8
// of head 2j + t/2) and the min term are added into the shared channel sums, which
// then go out with coalesced stores.
template <int G>
__device__ __forceinline__ void pv_flush(const GemvArgs& a, long bh, int warp, float* sacc,
                                         float (&acc_lo)[I8Layout<G>::kNH][8], float (&acc_hi)[I8Layout<G>::kNH][8],
                                         float (&mp)[G], int lane) {
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
  float* part = a.partials + (size_t)(warp + bh) * G * 128;
#pragma unroll
  for (int hd = 0; hd < G; ++hd) {
    const float mn = warp_sum(mp[hd]);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int c = sl * 32 + lane;
      __stcg(part + hd * 128 + c, sacc[hd * 128 + c] + mn);
    }
    mp[hd] = 0.f;
  }
  __syncwarp();
  zero_sums<G>(sacc, lane);
  __syncwarp();
}

// Warp whose item range holds `item` (ranges are [floor(w*N/W), floor((w+1)*N/W)), W <= N).
__device__ __forceinline__ long warp_of_item(long item, long n_items, long n_warps) {
  return (long)(((long long)(item + 1) * n_warps + n_items - 1) / n_items) - 1;
}

// Second pass of p·V: out = sum of the partials of every warp that touched
// (b, h), in a fixed order (deterministic).  One CTA per output row (b, h, head):
// warp i of 16 adds partial slots w0+i, w0+i+16, ... four independent 16-byte loads
// at a time (the partials sit in L2, so the time is latency, not bandwidth), then
// warp 0 adds the 16 warp sums in order.  It is launched as a programmatic
// dependent of pv_kernel and waits for its results.
constexpr int kReduceWarps = 16;

__device__ __forceinline__ void add4(float4& s, const float4 x) {
  s.x += x.x;
  s.y += x.y;
  s.z += x.z;
  s.w += x.w;
}

template <int G, class Plan>
__global__ void __launch_bounds__(kReduceWarps * 32)
    pv_reduce_kernel(const GemvArgs a, const __grid_constant__ Plan plan) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float4 warp_sum4[kReduceWarps][32];
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
  const long w0 = warp_of_item(first, a.n_items, a.n_warps) + bh;
  const long w1 = warp_of_item(first + n - 1, a.n_items, a.n_warps) + bh;
  const float4* base = reinterpret_cast<const float4*>(a.partials + hd * 128) + lane;
  const size_t slot_stride = (size_t)G * 128 / 4;  // float4 per partial slot
  constexpr long W = kReduceWarps;
  float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
  long w = w0 + warp;
  for (; w + 3 * W <= w1; w += 4 * W) {
    const float4 x0 = __ldcg(base + (size_t)w * slot_stride);
    const float4 x1 = __ldcg(base + (size_t)(w + W) * slot_stride);
    const float4 x2 = __ldcg(base + (size_t)(w + 2 * W) * slot_stride);
    const float4 x3 = __ldcg(base + (size_t)(w + 3 * W) * slot_stride);
    add4(s0, x0);
    add4(s1, x1);
    add4(s2, x2);
    add4(s3, x3);
  }
  for (; w <= w1; w += W) add4(s0, __ldcg(base + (size_t)w * slot_stride));
  add4(s0, s1);
  add4(s2, s3);
  add4(s0, s2);
  warp_sum4[warp][lane] = s0;
  __syncthreads();
  if (warp == 0) {
    float4 r = warp_sum4[0][lane];
#pragma unroll
    for (int i = 1; i < kReduceWarps; ++i) add4(r, warp_sum4[i][lane]);
    reinterpret_cast<float4*>(a.out + row * 128)[lane] = r;
  }
}

template <int BITS, int G, class Plan>
__global__ void __launch_bounds__(kWarpsPerCta * 32, pv_min_ctas(BITS, G))
    pv_kernel(const GemvArgs a, const __grid_constant__ Plan plan) {
  using C = Cfg<BITS, G, true>;
  extern __shared__ __align__(128) unsigned char smem[];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (warp >= a.n_warps) return;
  const WarpMem<BITS, G, true> m{smem + (threadIdx.x >> 5) * C::kWarpSmem};
  const long lo = (long)((long long)a.n_items * warp / a.n_warps);
  const long hi = (long)((long long)a.n_items * (warp + 1) / a.n_warps);
  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(m.bar(s), 1);
    fence_mbar_init();
  }
  __syncwarp();
  long prod = lo;
  Cursor pc = cursor_at(a, plan, lo);
  Cursor cc = pc;
  EntryWindow win;
  win.load(a, plan, lo, hi, lane);
  // p of the record in flight (this lane's slots 4*lane .. +3), loaded with its copy
  float4 pn[G];
  auto load_p = [&](const Cursor& c) {
    if (c.j < c.nb) {
      const long b = c.bh / a.kv_heads, h = c.bh % a.kv_heads;
      const float* prow = a.p + head_row(a, b, h, 0) * a.ld + (size_t)c.j * 128;
#pragma unroll
      for (int hd = 0; hd < G; ++hd) pn[hd] = __ldcs(reinterpret_cast<const float4*>(prow + hd * a.ld) + lane);
    }
  };
  for (int s0 = 0; s0 < C::kStages && prod < hi; ++s0, ++prod, cursor_next(a, plan, pc)) {
    issue_item<BITS, G, true>(a, m, pc, win.get(prod), s0, lane);
    if (!C::kStagedP) load_p(pc);
  }

  float mp[G];  // sum over the warp's records of p * mn (lane: slots 4*lane .. +3)
  float acc_lo[C::kNH][8], acc_hi[C::kNH][8];  // tensor-core path
#pragma unroll
  for (int hd = 0; hd < G; ++hd) mp[hd] = 0.f;
#pragma unroll
  for (int jn = 0; jn < C::kNH; ++jn)
#pragma unroll
    for (int T = 0; T < 8; ++T) acc_lo[jn][T] = acc_hi[jn][T] = 0.f;
  float* sacc = m.sums();
  zero_sums<G>(sacc, lane);
  __syncwarp();
  long cur_bh = cc.bh;
  uint32_t phases = 0;
  int s = 0;
  for (long x = lo; x < hi; ++x, cursor_next(a, plan, cc)) {
    const long bh = cc.bh;
    if (bh != cur_bh) {
      pv_flush<G>(a, cur_bh, warp, sacc, acc_lo, acc_hi, mp, lane);
      cur_bh = bh;
    }
    const bool ok = mbar_wait_bounded(m.bar(s), (phases >> s) & 1u, a.ctrl);
    phases ^= 1u << s;
    if (!ok) {
      drain_stages<BITS, G, true>(m, phases, s, x, prod, a.ctrl);
      return;
    }
    const int kind_len = *m.kind(s);
    const int kind = kind_len & 0xFF;
    unsigned char* st = m.stage(s);
    if (kind == kKindTail) {
      pv_tail<G>(a, bh, cc.nb, cc.tl, sacc, lane);
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
      float mpr[G];
#pragma unroll
      for (int hd = 0; hd < G; ++hd) {
        const float4 p4 = C::kStagedP ? reinterpret_cast<const float4*>(st + C::kStageRec + 512 * hd)[lane] : pn[hd];
        const float pr[4] = {p4.x, p4.y, p4.z, p4.w};
        mpr[hd] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mpr[hd] = fmaf(pr[i], mnr[i], mpr[hd]);
          pv4[hd][i] = pr[i] * scr[i];
        }
      }
      uint32_t* tab = m.table();
      float invf[G];
      build_i8tab<G, C::kNT>(tab, pv4, invf, lane);
      __syncwarp();
      bool ok = true;
      if (kind == kKindRaw)
        pv_i8<BITS, G>(st, tab, invf, acc_lo, acc_hi, lane);
      else
        ok = pv_packed_nat<BITS, G>(st, (uint32_t)(kind_len >> 8) * 16u, tab, invf, sacc, lane);
      if (ok) {
#pragma unroll
        for (int hd = 0; hd < G; ++hd) mp[hd] += mpr[hd];
      } else if (lane == 0) {
        set_status(a.ctrl, PACKKV_DEV_BAD_RECORD);
      }
    }
    __syncwarp();
    if (prod < hi) {
      if (prod - win.base >= 32) win.load(a, plan, prod, hi, lane);
      issue_item<BITS, G, true>(a, m, pc, win.get(prod), s, lane);
      if (!C::kStagedP) load_p(pc);
      ++prod;
      cursor_next(a, plan, pc);
    }
    s = (s + 1 == C::kStages) ? 0 : s + 1;
  }
  pv_flush<G>(a, cur_bh, warp, sacc, acc_lo, acc_hi, mp, lane);
}

// ----------------------------------------------------------------------------
// Host side: instantiation table, occupancy, launch
// ----------------------------------------------------------------------------
struct KernelInfo {
  const void* fn;
  int smem;
};

template <int BITS, int G, bool PV, class Plan>
KernelInfo kernel_info() {
  using C = Cfg<BITS, G, PV>;
  if constexpr (PV)
    return {reinterpret_cast<const void*>(&pv_kernel<BITS, G, Plan>), kWarpsPerCta * C::kWarpSmem};
  else
    return {reinterpret_cast<const void*>(&qk_kernel<BITS, G, Plan>), kWarpsPerCta * C::kWarpSmem};
}

template <bool PV, class Plan>
bool select(int bits, int group, KernelInfo* out) {
#define PACKKV_CASE(B, GG)                  \
  if (bits == B && group == GG) {           \
    *out = kernel_info<B, GG, PV, Plan>();  \
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

template <int G, class Plan>
const void* reduce_fn() {
  return reinterpret_cast<const void*>(&pv_reduce_kernel<G, Plan>);
}

template <bool PV, class Plan>
cudaError_t launch(GemvArgs a, const Plan* plan, cudaStream_t stream) {
  KernelInfo info{};
  if (!select<PV, Plan>(a.bits, a.group, &info)) return cudaErrorInvalidValue;
  int w = 0;
  cudaError_t e = resident_warps(info, &w);
  if (e != cudaSuccess) return e;
  if (w > gemv_max_warps()) w = gemv_max_warps();
  a.n_warps = (int)(a.n_items < w ? a.n_items : w);
  if (a.n_warps < 1) a.n_warps = 1;
  const unsigned grid = (unsigned)((a.n_warps + kWarpsPerCta - 1) / kWarpsPerCta);
  void* args[] = {&a, const_cast<Plan*>(plan)};
  if (a.n_items > 0) {
    e = cudaLaunchKernel(info.fn, dim3(grid), dim3(kWarpsPerCta * 32), args, info.smem, stream);
    if (e != cudaSuccess || !PV) return e;
  } else if (!PV) {
    return cudaSuccess;
  }
  // second pass of p·V, launched early (programmatic dependent launch); it waits for pv_kernel
  const long rows = (long)a.batch * a.kv_heads * a.group;
  const void* red = a.group == 1 ? reduce_fn<1, Plan>() : a.group == 2 ? reduce_fn<2, Plan>()
                  : a.group == 4 ? reduce_fn<4, Plan>() : reduce_fn<8, Plan>();
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(kReduceWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.n_items > 0 ? 1 : 0;
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
  if (!select<true, NoPlan>(a.bits, a.group, &info)) return cudaErrorInvalidValue;
  int w = 0;
  const cudaError_t e = resident_warps(info, &w);
  if (e != cudaSuccess) return e;
  if (w > gemv_max_warps()) w = gemv_max_warps();
  const long n_warps = a.n_items < w ? a.n_items : w;
  *bytes = ((size_t)n_warps + (size_t)a.batch * a.kv_heads) * a.group * 128 * sizeof(float);
  return cudaSuccess;
}

cudaError_t launch_qk(GemvArgs a, const RaggedPlan* plan, cudaStream_t stream) {
  static const NoPlan none{};
  return plan ? launch<false, RaggedPlan>(a, plan, stream) : launch<false, NoPlan>(a, &none, stream);
}
cudaError_t launch_pv(GemvArgs a, const RaggedPlan* plan, cudaStream_t stream) {
  static const NoPlan none{};
  return plan ? launch<true, RaggedPlan>(a, plan, stream) : launch<true, NoPlan>(a, &none, stream);
}

}  // namespace packkv
