// PackKV encoder: block quantization, joint token reorder, channel-direction
// bit-packing (packed-cache format v1, sections 1-4; PackKV paper page, Figure 2 steps (1)
// and (2), Figure 5 granularities, TL;DR).
//
// One encode call is one pass over the input: a CTA per (sequence, head, block)
// quantizes the K and V blocks, ranks the tokens, sizes the units, assembles both
// records in shared memory (while two warps find the arena offsets) and writes them
// at their arena offsets.  The offsets
// follow ascending (sequence, head, block) order, so they are prefix sums of
// the record lengths; a CTA learns its prefix by decoupled look-back over the
// index entries of the blocks before it:
//   * a CTA takes a ticket (the order in which CTAs started) and handles block
//     `ticket`, so every block before it belongs to a CTA that is running or done;
//   * once its lengths are known it publishes them in its index entries
//     ({length, AGGREGATE} in the {offset, length} words), then walks back until
//     it meets an entry that is final ({offset16, length16}: the prefix through
//     that block is offset16 - arena end + length16), summing the aggregates on
//     the way, and writes its own final entry;
//   * the last CTA to finish advances the arena ends, or, if any record did not
//     fit, marks every index entry of the call invalid and sets
//     PACKKV_DEV_CAPACITY (a record that did not fit was not written; records
//     that fit may have been written past the old arena end).
// Every wait (input copy, look-back) gives up after about a second, sets
// PACKKV_DEV_TIMEOUT and fails the call instead of hanging.
// The encoder runs once per 128 tokens per head; it is not on the per-token path.
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace packkv {

namespace {

constexpr uint32_t kFlagAggregate = 0x80000000u;  // {x = own length16, y = flag}: prefix not known yet
constexpr uint32_t kDone2 = 2u;                   // done counter step (bit 0: some record did not fit)
constexpr int kEncodeThreads = 512;
// storage-order code copies inside the (then unused) input buffers: above the first
// 12 KiB, which hold the record being assembled (at most 528 + 2048*4 bytes)
constexpr int kCodeCopyOffset = 12 * 1024;
constexpr int kVtPitch = 132;  // bytes per channel row of the transposed V codes (spreads banks)
static_assert(kCodeCopyOffset >= 528 + 2048 * 4, "records fit below the code copies");
static_assert(kCodeCopyOffset + 128 * kVtPitch <= 128 * 128 * 2, "code copies fit in an input buffer");
constexpr int kParts = kEncodeThreads / kBlockTokens;  // threads per channel / token in the reductions

struct EncodeSmem {  // two CTAs per SM: at most about 113 KB
  __half kx[kBlockTokens][kHeadDim];   // input K block; later the K record buffer
  __half vx[kBlockTokens][kHeadDim];   // input V block; later the V record buffer
  uint8_t ck[kBlockTokens][kHeadDim];  // K codes [token][channel] (first the range partials)
  uint8_t cv[kBlockTokens][kHeadDim];  // V codes [token][channel]
  uint16_t kmin[kHeadDim], kscale[kHeadDim];     // per channel
  uint16_t vmin[kBlockTokens], vscale[kBlockTokens];  // per token (original order)
  float krcp[kHeadDim];                          // 1 / scale (rounded), 0 for a zero scale
  float4 vq[kBlockTokens];  // per token: -min, 1 / scale (rounded, 0 for a zero scale), scale
  alignas(16) int key[kBlockTokens];  // reorder key * 128 + token
  int rank_part[kParts][kBlockTokens];
  uint8_t perm[kBlockTokens];          // perm[slot] = token
  uint8_t base[2][kGroups][kHeadDim];
  uint8_t width[2][kGroups][kHeadDim];
  uint16_t ustart[2][kGroups][kHeadDim];  // word index of each unit in the word area
  int group_total[2][kGroups];
  int wsum[2];
  int nonfinite;
  int failed;                          // this CTA's inputs or prefix could not be obtained
  int last;                            // this CTA finished last
  long ticket;
  unsigned long long prefix[2];        // exclusive prefix (16-byte units) of the K / V record
  uint64_t bar;
};

static_assert(sizeof(EncodeSmem) <= 113 * 1024, "two encoder CTAs per SM");

__device__ __forceinline__ int bitlen(uint32_t x) { return x == 0 ? 0 : 32 - __clz(x); }

constexpr float kEncRound = 12582912.0f;  // 1.5 * 2^23: y + kEncRound keeps rint(y) in the low bits

// The low bytes of four floats, packed in order.
__device__ __forceinline__ uint32_t low_bytes4(float2 lo, float2 hi) {
  return __byte_perm(__byte_perm(__float_as_uint(lo.x), __float_as_uint(lo.y), 0x0040u),
                     __byte_perm(__float_as_uint(hi.x), __float_as_uint(hi.y), 0x0040u), 0x5410u);
}

// code = clamp(rint(fl(d / s)), 0, qmax) for d = fl(x - mn) >= 0 and scale s > 0, with
// r = 1/s rounded to nearest.  q1 = fl(d * r) lies within 2^-18 of fl(d / s) (both are
// within 2^-19 of d / s, which is below 16), so the two round to the same integer unless
// fl(d / s) is within 2^-18 of a half-integer; then the correctly rounded quotient decides.
__device__ __forceinline__ int quant_code(float d, float s, float r, int qmax) {
  const float q1 = __fmul_rn(d, r);
  const float h = __fsub_rn(__fsub_rn(q1, floorf(q1)), 0.5f);  // exact
  const float y = fabsf(h) > 7.62939453125e-06f ? q1 : __fdiv_rn(d, s);  // 2^-17
  return (int)fminf(fmaxf(rintf(y), 0.0f), (float)qmax);
}

// Where block t of the call goes: the index entry (u32 pair index) of its (sequence,
// head, logical block) -- through the block table if the cache has one -- and the row of
// the input it is read from.  Uniform calls cover every sequence; ragged calls the
// plan's sequences, each from its own first logical block.
struct CallBlock {
  size_t entry;  // u32 pair index into the index table
  size_t row;    // input row: ((sequence * heads + head) * nb + i)
};

template <class Plan>
__device__ __forceinline__ CallBlock call_block(const EncodeArgs& a, const Plan& plan, long t) {
  const long i = t % a.nb, sh = t / a.nb;  // sh = (sequence of the call) * heads + head
  const long h = sh % a.heads;
  long b, j;
  if constexpr (std::is_same<Plan, RaggedEncodePlan>::value) {
    const long sidx = sh / a.heads;
    b = plan.seq[sidx];
    j = plan.first_block[sidx] + i;
  } else {
    b = sh / a.heads;
    j = a.n_old + i;
  }
  long rb = b, jb = j;
  if (a.block_table != nullptr) {
    const int p = a.block_table[(size_t)b * a.max_blocks + j];
    rb = p / a.max_blocks;
    jb = p % a.max_blocks;
  }
  CallBlock c;
  c.entry = ((size_t)rb * a.heads + h) * a.max_blocks + jb;
  c.row = ((size_t)b * a.heads + h) * a.nb + i;
  return c;
}

template <class Plan>
__device__ __forceinline__ unsigned long long* entry64(uint32_t* index, const EncodeArgs& a, const Plan& plan,
                                                       long blk_in_call) {
  return reinterpret_cast<unsigned long long*>(index + call_block(a, plan, blk_in_call).entry * 2);
}

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Exclusive prefix, in 16-byte units, of block `t` of the call for one tensor, by
// look-back over the entries of blocks t-1, t-2, ..., 32 at a time (one warp, lane
// l reading block p - l).  Within a window, the nearest final entry ends the walk
// (its prefix plus the aggregates above it); a window without one adds its 32
// aggregates and moves down.  A window waits while any entry above its nearest
// final entry is unpublished.  Returns false (and sets PACKKV_DEV_TIMEOUT) if a
// predecessor did not publish within about a second.
template <class Plan>
__device__ bool look_back(uint32_t* index, const EncodeArgs& a, const Plan& plan, long t, unsigned long long end0,
                          unsigned long long* excl, int lane) {
  unsigned long long sum = 0;
  long p = t - 1;  // top of the current window
  uint64_t start = 0;
  uint32_t it = 0;
  while (p >= 0) {
    const long mine = p - lane;
    unsigned long long e = 0;
    if (mine >= 0) e = ld_relaxed(entry64(index, a, plan, mine));
    const uint32_t y = (uint32_t)(e >> 32);
    const bool unpublished = mine >= 0 && y == 0u;
    const bool fin = mine >= 0 && y != 0u && !(y & kFlagAggregate);
    const uint32_t fin_mask = __ballot_sync(0xffffffffu, fin);
    const uint32_t unp_mask = __ballot_sync(0xffffffffu, unpublished);
    // lanes above (nearer to t than) the nearest final entry must all be published
    const int stop = fin_mask ? __ffs(fin_mask) - 1 : 32;  // lowest lane = nearest block
    const uint32_t need = stop >= 32 ? 0xffffffffu : ((1u << stop) - 1u);
    if (unp_mask & need) {
      if (start == 0) start = global_ns();
      if ((++it & 63u) == 0u && global_ns() - start > 1000000000ull) {
        if (lane == 0) set_status(a.ctrl, PACKKV_DEV_TIMEOUT);
        *excl = sum;
        return false;
      }
      continue;
    }
    unsigned long long v = 0;
    if (mine >= 0 && lane < stop) v = (uint32_t)e;                                  // aggregates
    if (lane == stop) v = (unsigned long long)(uint32_t)e - end0 + y;               // final: prefix
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    sum += v;
    if (stop < 32) break;
    p -= 32;
  }
  *excl = sum;
  return true;
}

template <class Plan>
__global__ void __launch_bounds__(kEncodeThreads) encode_kernel(const EncodeArgs a, const __grid_constant__ Plan plan) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EncodeSmem& s = *reinterpret_cast<EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int qmax = (1 << a.bits) - 1;
  const long n_call = (long)a.batch * a.heads * a.nb;
  unsigned int* counters = reinterpret_cast<unsigned int*>(a.ctrl + kCtrlScratch);  // [ticket, done]

  // ---- ticket, then both input blocks by bulk copy ---------------------------
  if (tid == 0) {
    s.ticket = (long)atomicAdd(&counters[0], 1u);
    s.nonfinite = 0;
    s.failed = 0;
    s.wsum[0] = s.wsum[1] = 0;
    mbar_init(&s.bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const long t_call = s.ticket;                 // block index within the call
  const CallBlock where = call_block(a, plan, t_call);
  const size_t in_base = where.row * kBlockTokens * kHeadDim;
  const size_t slot = where.entry;  // the block's index entry (and its row of perm)
  if (tid == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&s.bar, 2u * kBlockTokens * kHeadDim * 2u);
    bulk_g2s(&s.kx[0][0], a.k + in_base, kBlockTokens * kHeadDim * 2u, &s.bar);
    bulk_g2s(&s.vx[0][0], a.v + in_base, kBlockTokens * kHeadDim * 2u, &s.bar);
  }
  const bool input_ok = mbar_wait_bounded(&s.bar, 0u, a.ctrl);
  if (!input_ok) s.failed = 1;  // every writer writes 1
  __syncthreads();

  // ---- quantization ranges (K per channel, V per token) and non-finite values ---
  // fp16 pairs: min / max of fp16 values are exact in fp16 (a signed zero is normalised
  // below).  The NaN-propagating forms carry a NaN, and min / max carry an infinity, to
  // the slice results, so one test of those finds every non-finite input: a value whose
  // exponent field is all ones carries into bit 15 of its half when 0x0400 is added.
  {
    const __half2* k2 = reinterpret_cast<const __half2*>(&s.kx[0][0]);  // [token][channel pair]
    const __half2* v2 = reinterpret_cast<const __half2*>(&s.vx[0][0]);
    constexpr int kPairs = kHeadDim / 2;
    constexpr int kKParts = kEncodeThreads / kPairs;      // token slices per K channel pair
    constexpr int kKSlice = kBlockTokens / kKParts;
    constexpr int kVSlice = kPairs / kParts;              // channel pairs per V token slice
    const int cp = tid % kPairs, kpart = tid / kPairs;
    const int t = tid % kBlockTokens, vpart = tid / kBlockTokens;
    __half2 kmn = k2[kKSlice * kpart * kPairs + cp], kmx = kmn;
#pragma unroll 8
    for (int i = 0; i < kKSlice; ++i) {
      const __half2 h = k2[(kKSlice * kpart + i) * kPairs + cp];
      kmn = __hmin2_nan(kmn, h);
      kmx = __hmax2_nan(kmx, h);
    }
    // a token's pairs from a rotated start: the 32 tokens of a warp hit 32 banks
    const int p0 = kVSlice * vpart + t;
    __half2 vmn = v2[t * kPairs + (p0 & (kPairs - 1))], vmx = vmn;
#pragma unroll 8
    for (int j = 0; j < kVSlice; ++j) {
      const __half2 h = v2[t * kPairs + ((p0 + j) & (kPairs - 1))];
      vmn = __hmin2_nan(vmn, h);
      vmx = __hmax2_nan(vmx, h);
    }
    auto nonfinite2 = [](__half2 x) {
      return ((*reinterpret_cast<const uint32_t*>(&x) & 0x7C007C00u) + 0x04000400u) & 0x80008000u;
    };
    const uint32_t bad = nonfinite2(kmn) | nonfinite2(kmx) | nonfinite2(vmn) | nonfinite2(vmx);
    __half2* redk = reinterpret_cast<__half2*>(&s.ck[0][0]);  // [min, max][kKParts][kPairs]
    __half* redv = reinterpret_cast<__half*>(&s.ck[0][0]) + 2 * 2 * kEncodeThreads;  // [min, max][kParts][128]
    redk[kpart * kPairs + cp] = kmn;
    redk[(kKParts + kpart) * kPairs + cp] = kmx;
    redv[vpart * kBlockTokens + t] = __hmin(__low2half(vmn), __high2half(vmn));
    redv[(kParts + vpart) * kBlockTokens + t] = __hmax(__low2half(vmx), __high2half(vmx));
    if (bad) s.nonfinite = 1;
  }
  __syncthreads();
  if (tid == 0 && s.nonfinite) set_status(a.ctrl, PACKKV_DEV_NONFINITE);
  if (tid < 2 * kBlockTokens) {
    const bool is_k = tid < kBlockTokens;
    const int i = tid % kBlockTokens;
    // K: the halves of channel i over the token slices; V: token i over the pair slices
    const __half* red = reinterpret_cast<const __half*>(&s.ck[0][0]) + (is_k ? 0 : 2 * 2 * kEncodeThreads);
    const int nq = is_k ? kEncodeThreads / (kHeadDim / 2) : kParts;
    __half hlo = red[i], hhi = red[nq * kBlockTokens + i];
    for (int q = 1; q < nq; ++q) {
      hlo = __hmin(hlo, red[q * kBlockTokens + i]);
      hhi = __hmax(hhi, red[(nq + q) * kBlockTokens + i]);
    }
    float lo = __half2float(hlo);
    const float hi = __half2float(hhi);
    if (lo == 0.0f) lo = 0.0f;  // -0 is stored as +0
    const float range = __fsub_rn(hi, lo);
    uint16_t sc = 0;
    if (range > 0.0f) sc = __half_as_ushort(__float2half_ru(__fdiv_rn(range, (float)qmax)));
    const uint16_t mnb = __half_as_ushort(__float2half_rn(lo));  // exact: lo is an fp16 value
    const float rcp = sc ? __frcp_rn(half_bits_to_float(sc)) : 0.0f;
    if (is_k) {
      s.kmin[i] = mnb;
      s.kscale[i] = sc;
      s.krcp[i] = rcp;
    } else {
      s.vmin[i] = mnb;
      s.vscale[i] = sc;
      s.vq[i] = make_float4(-half_bits_to_float(mnb), rcp, half_bits_to_float(sc), 0.0f);
    }
  }
  __syncthreads();

  // ---- codes and reorder keys ---------------------------------------------------
  // A thread keeps four channels (their K parameters in registers) and walks tokens;
  // the four codes of a tensor go to shared memory as one word, and a warp's 32 lanes
  // (all channels of one token) sum the token's reorder key.  Fast path in pairs:
  // q = fl(x - mn) * RN(1/scale), rint(q) by adding and removing 1.5 * 2^23 (ties to
  // even), e = q - rint(q) exactly.  quant_code takes the correctly rounded quotient
  // where it can differ, |e| >= 0.5 - 2^-17; where q is not finite or not below
  // qmax + 0.5 (no clamp needed on the fast path), it takes the element too.
  {
    static_assert(kEncodeThreads % (kHeadDim / 4) == 0, "a thread keeps its channels");
    constexpr int kQuads = kHeadDim / 4, kRows = kEncodeThreads / kQuads;
    const int j = tid % kQuads;
    const float2 R = make_float2(kEncRound, kEncRound), nR = make_float2(-kEncRound, -kEncRound);
    const float lim = (float)qmax + 0.5f;
    constexpr float kTie = 0.5f - 7.62939453125e-06f;  // 0.5 - 2^-17
    float2 nkmn[2], kr[2];
    float ksc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ksc[i] = half_bits_to_float(s.kscale[4 * j + i]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      nkmn[h] = make_float2(-half_bits_to_float(s.kmin[4 * j + 2 * h]), -half_bits_to_float(s.kmin[4 * j + 2 * h + 1]));
      kr[h] = make_float2(s.krcp[4 * j + 2 * h], s.krcp[4 * j + 2 * h + 1]);
    }
    // the four codes of x[0..3] (pairs x[h]) for minus-min nm, reciprocals r, scales sc
    auto codes4 = [&](const float2 (&x)[2], const float2 (&nm)[2], const float2 (&r)[2],
                      const float (&sc)[4]) -> uint32_t {
      float2 d[2], q[2], u[2];
      bool fast = true;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        d[h] = __fadd2_rn(x[h], nm[h]);
        q[h] = __fmul2_rn(d[h], r[h]);
        u[h] = __fadd2_rn(q[h], R);
        const float2 e = __ffma2_rn(__fadd2_rn(u[h], nR), make_float2(-1.f, -1.f), q[h]);  // exact
        fast = fast && q[h].x < lim && q[h].y < lim && fabsf(e.x) < kTie && fabsf(e.y) < kTie;
      }
      if (fast) return low_bytes4(u[0], u[1]);  // of 1.5 * 2^23 + rint(q): rint(q)
      uint32_t w = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float di = (i & 1) ? d[i >> 1].y : d[i >> 1].x;
        const float ri = (i & 1) ? r[i >> 1].y : r[i >> 1].x;
        const int c = sc[i] > 0.0f ? quant_code(di, sc[i], ri, qmax) : 0;
        w |= (uint32_t)c << (8 * i);
      }
      return w;
    };
    for (int t = tid / kQuads; t < kBlockTokens; t += kRows) {
      const uint2 kw = *reinterpret_cast<const uint2*>(&s.kx[t][4 * j]);
      const float2 xk[2] = {__half22float2(*reinterpret_cast<const __half2*>(&kw.x)),
                            __half22float2(*reinterpret_cast<const __half2*>(&kw.y))};
      const uint32_t kcodes = codes4(xk, nkmn, kr, ksc);
      *reinterpret_cast<uint32_t*>(&s.ck[t][4 * j]) = kcodes;
      const uint2 vw = *reinterpret_cast<const uint2*>(&s.vx[t][4 * j]);
      const float2 xv[2] = {__half22float2(*reinterpret_cast<const __half2*>(&vw.x)),
                            __half22float2(*reinterpret_cast<const __half2*>(&vw.y))};
      const float4 pq = s.vq[t];
      const float nvm = pq.x, vr = pq.y, vs = pq.z;
      const float2 nvm2[2] = {make_float2(nvm, nvm), make_float2(nvm, nvm)};
      const float2 vr2[2] = {make_float2(vr, vr), make_float2(vr, vr)};
      const float vsc[4] = {vs, vs, vs, vs};
      const uint32_t vcodes = codes4(xv, nvm2, vr2, vsc);
      *reinterpret_cast<uint32_t*>(&s.cv[t][4 * j]) = vcodes;
      // the reorder key of token t (the warp holds all its channels): the sum of its K
      // codes (plus its V codes for the K+V key), then the token index below it, so
      // that all keys differ and a plain count gives the stable rank
      uint32_t sum = 0u;
      if (a.key_kind != PACKKV_KEY_IDENTITY) {
        sum = __dp4a(kcodes, 0x01010101u, 0u);
        if (a.key_kind == PACKKV_KEY_KV_SUM) sum = __dp4a(vcodes, 0x01010101u, sum);
      }
      sum = __reduce_add_sync(0xffffffffu, sum);
      if (j == 0) s.key[t] = (int)sum * kBlockTokens + t;
    }
  }
  __syncthreads();

  // ---- stable rank -------------------------------------------------------------
  {
    // rank of token t = #{u : key[u] < key[t] or (key[u] == key[t] and u < t)}: with the
    // index below the key (key * 128 + u), #{u : composite[u] < composite[t]};
    // kParts threads per token, each counting over a slice of the tokens
    constexpr int kSlice = kBlockTokens / kParts;
    const int t = tid % kBlockTokens, part = tid / kBlockTokens;
    const int kt = s.key[t];
    const int4* k4 = reinterpret_cast<const int4*>(&s.key[kSlice * part]);
    int r = 0;
#pragma unroll
    for (int i = 0; i < kSlice / 4; ++i) {
      const int4 ku = k4[i];
      r += (ku.x < kt) + (ku.y < kt) + (ku.z < kt) + (ku.w < kt);
    }
    s.rank_part[part][t] = r;
  }
  __syncthreads();
  if (tid < kBlockTokens) {
    int r = 0;
#pragma unroll
    for (int q = 0; q < kParts; ++q) r += s.rank_part[q][tid];
    s.perm[r] = (uint8_t)tid;
  }
  __syncthreads();

  // ---- codes in storage order, for the fragment words of raw records ----------
  // K: kp[slot][channel] (row copies); V: vt[channel][slot] (transposed, pitch 132).
  // Both live in the input buffers, which the codes no longer need, above the part
  // that later holds the records.
  uint8_t* kp = reinterpret_cast<uint8_t*>(&s.kx[0][0]) + kCodeCopyOffset;
  uint8_t* vt = reinterpret_cast<uint8_t*>(&s.vx[0][0]) + kCodeCopyOffset;
  for (int i = tid; i < kBlockTokens * kHeadDim / 16; i += blockDim.x) {
    const int r = i >> 3, q = i & 7;
    reinterpret_cast<uint4*>(kp + r * kHeadDim)[q] = reinterpret_cast<const uint4*>(s.ck[s.perm[r]])[q];
  }
  // V: four slots x four channels per task, a 4x4 byte transpose of four row words
  for (int i = tid; i < kHeadDim * kBlockTokens / 16; i += blockDim.x) {
    const int cq = i & (kHeadDim / 4 - 1), r4 = (i >> 5) * 4;  // lanes take consecutive channel quads
    const uint32_t w0 = reinterpret_cast<const uint32_t*>(s.cv[s.perm[r4]])[cq];
    const uint32_t w1 = reinterpret_cast<const uint32_t*>(s.cv[s.perm[r4 + 1]])[cq];
    const uint32_t w2 = reinterpret_cast<const uint32_t*>(s.cv[s.perm[r4 + 2]])[cq];
    const uint32_t w3 = reinterpret_cast<const uint32_t*>(s.cv[s.perm[r4 + 3]])[cq];
    const uint32_t lo01 = __byte_perm(w0, w1, 0x5140u), hi01 = __byte_perm(w0, w1, 0x7362u);  // b0 b4 b1 b5 / b2 b6 b3 b7
    const uint32_t lo23 = __byte_perm(w2, w3, 0x5140u), hi23 = __byte_perm(w2, w3, 0x7362u);
    uint8_t* dst = vt + 4 * cq * kVtPitch + r4;
    *reinterpret_cast<uint32_t*>(dst) = __byte_perm(lo01, lo23, 0x5410u);                // channel 4cq
    *reinterpret_cast<uint32_t*>(dst + kVtPitch) = __byte_perm(lo01, lo23, 0x7632u);     // 4cq + 1
    *reinterpret_cast<uint32_t*>(dst + 2 * kVtPitch) = __byte_perm(hi01, hi23, 0x5410u); // 4cq + 2
    *reinterpret_cast<uint32_t*>(dst + 3 * kVtPitch) = __byte_perm(hi01, hi23, 0x7632u); // 4cq + 3
  }

  __syncthreads();  // the storage-order copies are complete

  // code of storage slot r, channel c: K from the row copies, V from the transposed ones
  auto slot_code = [&](int tensor, int r, int c) -> int {
    return tensor ? vt[c * kVtPitch + r] : kp[r * kHeadDim + c];
  };

  // ---- frame of reference and width of every (group, channel) unit ----------
  for (int u = tid; u < 2 * kGroups * kHeadDim; u += blockDim.x) {
    const int tensor = u >> 9, g = (u >> 7) & 3, c = u & 127;
    int lo = 255, hi = 0;
#pragma unroll 8
    for (int j = 0; j < kGroupTokens; ++j) {
      const int code = slot_code(tensor, g * kGroupTokens + j, c);
      lo = min(lo, code);
      hi = max(hi, code);
    }
    if (a.unit_mode == (int)PACKKV_UNITS_WIDTH_ONLY) lo = 0;  // no frame of reference
    const int w = bitlen((uint32_t)(hi - lo));
    s.base[tensor][g][c] = (uint8_t)lo;
    s.width[tensor][g][c] = (uint8_t)w;
    // a warp's 32 units belong to one tensor (512 units per tensor, warps of 32)
    const int wsum = (int)__reduce_add_sync(0xffffffffu, (unsigned)w);
    if ((tid & 31) == 0) atomicAdd(&s.wsum[tensor], wsum);
  }
  __syncthreads();

  // raw fallback: the compressed record must be strictly smaller than the raw one
  const int raw_bytes = raw_record_bytes(a.bits);
  int rec_bytes[2];
  bool raw[2];
#pragma unroll
  for (int tensor = 0; tensor < 2; ++tensor) {
    const int packed = (1040 + 4 * s.wsum[tensor] + 15) & ~15;
    raw[tensor] = packed >= raw_bytes;
    rec_bytes[tensor] = raw[tensor] ? raw_bytes : packed;
  }

  // ---- publish the lengths (look-back aggregates) ---------------------------
  if (tid == 0 || tid == 32) {
    const int tensor = tid >> 5;
    uint32_t* index = tensor ? a.v_index : a.k_index;
    const unsigned long long agg =
        (unsigned long long)(uint32_t)(rec_bytes[tensor] >> 4) | ((unsigned long long)kFlagAggregate << 32);
    atomicExch(entry64(index, a, plan, t_call), agg);
  }

  // ---- unit word offsets ------------------------------------------------------
  if (tid < 256) {
    const int warp = tid >> 5, lane = tid & 31;  // warps 0..7 = (tensor, group)
    const int tensor = warp >> 2, g = warp & 3;
    int w4[4];
    int local = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w4[i] = raw[tensor] ? a.bits : s.width[tensor][g][lane * 4 + i];
      local += w4[i];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int at = incl - local;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s.ustart[tensor][g][lane * 4 + i] = (uint16_t)at;
      at += w4[i];
    }
    if (lane == 31) s.group_total[tensor][g] = incl;
  }
  __syncthreads();

  // ---- look-back: arena offsets (warp 0: K, warp 1: V), while warps 2.. assemble ----
  if (tid < 64) {
    const int tensor = tid >> 5, lane = tid & 31;
    uint32_t* index = tensor ? a.v_index : a.k_index;
    const unsigned long long end0 = a.ctrl[tensor ? kCtrlVEnd : kCtrlKEnd];
    unsigned long long excl = 0;
    const bool ok = look_back(index, a, plan, t_call, end0, &excl, lane);
    if (lane == 0) {
      if (!ok) s.failed = 1;
      s.prefix[tensor] = excl;
      // final entry {offset16, length16}; a failed call is invalidated by the last CTA
      const unsigned long long fin = (unsigned long long)(uint32_t)(end0 + excl) |
                                     ((unsigned long long)(uint32_t)(rec_bytes[tensor] >> 4) << 32);
      atomicExch(entry64(index, a, plan, t_call), fin);
    }
  }
  // ---- assemble both records in shared memory (reusing the input buffers) ---
  // Threads 64.. (asm = tid - 64) write every byte of both records: header, parameters,
  // meta, each word by exactly one thread, and the zero padding to 16 bytes.
  uint32_t* rec32[2] = {reinterpret_cast<uint32_t*>(&s.kx[0][0]), reinterpret_cast<uint32_t*>(&s.vx[0][0])};
  constexpr int kAsmFirst = 64;
  const int asm_id = tid - kAsmFirst, n_asm = (int)blockDim.x - kAsmFirst;
#pragma unroll
  for (int tensor = 0; tensor < 2; ++tensor) {
    unsigned char* rec = reinterpret_cast<unsigned char*>(rec32[tensor]);
    if (asm_id == 0) {
      uint16_t* gws = reinterpret_cast<uint16_t*>(rec);
      int acc = 0;
      for (int g = 0; g < kGroups; ++g) {
        gws[g] = (uint16_t)acc;
        acc += s.group_total[tensor][g];
      }
      const uint32_t flags = (raw[tensor] ? kRawFlag : 0u) | (tensor ? kVFlag : 0u) |
                             (PACKKV_FORMAT_VERSION << 8) | ((uint32_t)a.bits << 16);
      reinterpret_cast<uint32_t*>(rec)[2] = flags;
      reinterpret_cast<uint32_t*>(rec)[3] = (uint32_t)acc;
      // zero padding after the last word (compressed records; raw ones end on 16 bytes)
      const int end_words = (raw[tensor] ? kRawWordOffset / 4 + 512 * a.bits : kPackedWordOffset / 4 + acc);
      for (int wpad = end_words; wpad < rec_bytes[tensor] / 4; ++wpad) rec32[tensor][wpad] = 0u;
    }
    if (asm_id >= 0 && asm_id < kHeadDim) {
      uint16_t* mn = reinterpret_cast<uint16_t*>(rec + kParamOffset);
      uint16_t* sc = mn + kHeadDim;
      if (tensor == 0) {
        mn[asm_id] = s.kmin[asm_id];
        sc[asm_id] = s.kscale[asm_id];
      } else {
        mn[asm_id] = s.vmin[s.perm[asm_id]];
        sc[asm_id] = s.vscale[s.perm[asm_id]];
      }
    }
    if (!raw[tensor] && asm_id >= 0) {
      for (int u = asm_id; u < kGroups * kHeadDim; u += n_asm) {
        const int g = u >> 7, c = u & 127;
        rec[kMetaOffset + u] = (uint8_t)(s.base[tensor][g][c] | (s.width[tensor][g][c] << 4));
      }
    }
  }
  // raw records: words in 8-bit tensor-core fragment order (packed-cache format v1, section 4).
  // A[m][k] = code of slot m, channel k (K: kp row m) or of slot k, channel m (V: vt row
  // m).  A word's byte e holds column k0 + e of rows (16T + 8rh + g): one 32-bit load
  // of a storage-order row gives the four codes of a (row, byte) field set, placed by
  // one shift.  b = 3: bits 0-1 in words 0..1023 (the b = 2 order), bit 2 in 1024..1535.
  // Word wj = ((row group * 2 + J) * 32 + 4g + t) * 4 + 2 Q2 + kh, kappa = 2J + Q2; the row
  // group is the tile (b = 4), the tile pair (b = 2, low plane of b = 3) or the tile quad
  // (bit-2 plane).  A task is one (row group, J, t, Q2, kh) and walks g = 0..7: the lanes
  // of a warp then read 32 different banks.
  {
    const int n_tasks = 512 * a.bits / 8;  // per tensor
    for (int task = asm_id; asm_id >= 0 && task < 2 * n_tasks; task += n_asm) {
      const int tensor = task >= n_tasks ? 1 : 0;
      if (!raw[tensor]) continue;
      const int tk = task - tensor * n_tasks;
      uint32_t* words = rec32[tensor] + kRawWordOffset / 4;
      const uint8_t* rows = tensor ? vt : kp;
      const int pitch = tensor ? kVtPitch : kHeadDim;
      const bool plane1 = a.bits == 3 && tk >= 128;
      const int tj = plane1 ? tk - 128 : tk;
      const int i = tj & 3, t = (tj >> 2) & 3, jj = (tj >> 4) & 1, tp = tj >> 5;
      const uint8_t* col = rows + 32 * (2 * jj + (i >> 1)) + 16 * (i & 1) + 4 * t;
      uint32_t* wout = words + (plane1 ? 1024 : 0) + ((tp * 2 + jj) * 32 + t) * 4 + i;
#pragma unroll 2
      for (int g = 0; g < 8; ++g, col += pitch) {
        auto row4 = [&](int m8) { return *reinterpret_cast<const uint32_t*>(col + m8 * 8 * pitch); };
        uint32_t word;
        if (a.bits == 4) {
          word = row4(2 * tp) | (row4(2 * tp + 1) << 4);  // rows 16T + g, 16T + 8 + g
        } else if (!plane1) {
          const uint32_t m3 = a.bits == 3 ? 0x03030303u : 0xFFFFFFFFu;
          word = (row4(4 * tp) & m3) | ((row4(4 * tp + 1) & m3) << 2) | ((row4(4 * tp + 2) & m3) << 4) |
                 ((row4(4 * tp + 3) & m3) << 6);
        } else {
          word = 0u;
#pragma unroll
          for (int sg = 0; sg < 8; ++sg) word |= ((row4(8 * tp + sg) >> 2) & 0x01010101u) << sg;
        }
        wout[16 * g] = word;
      }
    }
  }
  // pack the units: every word is owned by exactly one thread.  A unit's 32 offsets are
  // held as eight words of four bytes (slots 4k .. 4k+3 in word k); each slice is then
  // gathered with shifts, masks and byte permutes (field j of a p-bit slice at bit
  // (j p) mod 32 of word (j p) / 32, packed-cache format v1, section 3).
  for (int u = asm_id; asm_id >= 0 && u < 2 * kGroups * kHeadDim; u += n_asm) {
    const int tensor = u >> 9, g = (u >> 7) & 3, c = u & 127;
    if (raw[tensor]) continue;  // written above
    const int w = s.width[tensor][g][c];
    if (w == 0) continue;
    const uint32_t base4 = (uint32_t)s.base[tensor][g][c] * 0x01010101u;
    int gstart = 0;
    for (int gg = 0; gg < g; ++gg) gstart += s.group_total[tensor][gg];
    uint32_t* words = rec32[tensor] + kPackedWordOffset / 4 + gstart + s.ustart[tensor][g][c];
    uint32_t ow[8];  // offsets (code - base, no borrow between bytes)
    if (tensor) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(vt + c * kVtPitch + g * kGroupTokens);
#pragma unroll
      for (int k = 0; k < 8; ++k) ow[k] = src[k] - base4;
    } else {
      const uint8_t* src = kp + g * kGroupTokens * kHeadDim + c;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t b0 = src[(4 * k) * kHeadDim], b1 = src[(4 * k + 1) * kHeadDim];
        const uint32_t b2 = src[(4 * k + 2) * kHeadDim], b3 = src[(4 * k + 3) * kHeadDim];
        ow[k] = __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u) - base4;
      }
    }
    // slices in descending size: 4 | 2 then 1 | 2 | 1
    int at = 0, lo = 0;
    if (w == 4) {  // word q: slots 8q .. 8q+7, a nibble each
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t y0 = ow[2 * q] | (ow[2 * q] >> 4), y1 = ow[2 * q + 1] | (ow[2 * q + 1] >> 4);
        words[q] = __byte_perm(y0, y1, 0x6420u);
      }
      at = 4;
    }
    if (w & 2) {  // word q: slots 16q .. 16q+15, two bits each, from bits 0-1
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t z[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t x = ow[4 * q + k] & 0x03030303u;
          const uint32_t y = x | (x >> 6);  // bytes 0 and 2: two fields each
          z[k] = y | (y >> 12);             // byte 0: slots 4k .. 4k+3
        }
        words[at + q] = __byte_perm(__byte_perm(z[0], z[1], 0x0040u), __byte_perm(z[2], z[3], 0x0040u), 0x5410u);
      }
      at += 2;
      lo = 2;
    }
    if (w & 1) {  // one word: slot j at bit j, from bit lo
      uint32_t word = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t x = (ow[k] >> lo) & 0x01010101u;
        word |= ((x * 0x10204080u) >> 28) << (4 * k);  // bit of byte e -> bit 28 + e
      }
      words[at] = word;
    }
  }

  __syncthreads();  // records assembled, arena offsets known

  // ---- write the records that fit and the permutation ------------------------
  bool fits_all = !s.failed;
#pragma unroll
  for (int tensor = 0; tensor < 2; ++tensor) {
    uint8_t* arena = tensor ? a.v_arena : a.k_arena;
    const unsigned long long off16 = a.ctrl[tensor ? kCtrlVEnd : kCtrlKEnd] + s.prefix[tensor];
    const bool fits =
        !s.failed && (off16 + (unsigned long long)(rec_bytes[tensor] >> 4)) * 16ull <= a.arena_bytes;
    fits_all = fits_all && fits;
    if (!fits) continue;
    uint4* dst = reinterpret_cast<uint4*>(arena + off16 * 16);
    const uint4* src = reinterpret_cast<const uint4*>(rec32[tensor]);
    for (int i = tid; i < rec_bytes[tensor] / 16; i += blockDim.x) dst[i] = src[i];
  }
  if (a.perm != nullptr && tid < kBlockTokens) a.perm[slot * kBlockTokens + tid] = s.perm[tid];
  __syncthreads();

  // ---- completion: the last CTA advances the arena ends or fails the call ----
  if (tid == 0) {
    __threadfence();
    const unsigned int mine = kDone2 | (fits_all ? 0u : 1u);
    const unsigned int prev = atomicAdd(&counters[1], mine);
    s.last = (long)(prev >> 1) == n_call - 1;
    if (s.last) {
      __threadfence();
      s.failed = (int)((prev | mine) & 1u);
    }
  }
  __syncthreads();
  // a copy that did not land in time: give it one more bounded wait before exiting
  if (!input_ok && tid == 0) mbar_wait_bounded(&s.bar, 0u, a.ctrl);
  if (!s.last) return;
  if (s.failed) {
    for (long e = tid; e < n_call; e += blockDim.x) {
      *entry64(a.k_index, a, plan, e) = 0xFFFFFFFFull;  // {offset 0xFFFFFFFF, length 0}
      *entry64(a.v_index, a, plan, e) = 0xFFFFFFFFull;
    }
    if (tid == 0) set_status(a.ctrl, PACKKV_DEV_CAPACITY);
  } else if (tid == 0 || tid == 32) {
    // prefix through the last block of the call = its final entry's offset - end + length
    const int tensor = tid >> 5;
    uint32_t* index = tensor ? a.v_index : a.k_index;
    const unsigned long long e = atomicAdd(entry64(index, a, plan, n_call - 1), 0ull);
    const unsigned long long end0 = a.ctrl[tensor ? kCtrlVEnd : kCtrlKEnd];
    const unsigned long long total = (unsigned long long)(uint32_t)e - end0 + (uint32_t)(e >> 32);
    a.ctrl[tensor ? kCtrlVEnd : kCtrlKEnd] = end0 + total;
  }
  __syncthreads();
  if (tid == 0) a.ctrl[kCtrlScratch] = 0ull;  // ticket and done counters for the next call
}

// Copies one token per (sequence, head) into the tail at position `pos`.
__global__ void append_tail_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                   uint16_t* __restrict__ k_tail, uint16_t* __restrict__ v_tail, int n_bh,
                                   int pos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // 16-byte chunk
  const int per_bh = kHeadDim * 2 / 16;                  // 16 chunks per token
  if (i >= 2 * n_bh * per_bh) return;
  const int tensor = i / (n_bh * per_bh);
  const int r = i % (n_bh * per_bh);
  const int bh = r / per_bh, ch = r % per_bh;
  const uint4* src = reinterpret_cast<const uint4*>((tensor ? v : k) + (size_t)bh * kHeadDim);
  uint4* dst = reinterpret_cast<uint4*>((tensor ? v_tail : k_tail) + ((size_t)bh * kBlockTokens + pos) * kHeadDim);
  dst[ch] = src[ch];
}

// As append_tail_kernel, with each sequence's own position (plan.pos[b]; none if < 0).
__global__ void append_tail_ragged_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                          uint16_t* __restrict__ k_tail, uint16_t* __restrict__ v_tail, int batch,
                                          int heads, const __grid_constant__ RaggedAppendPlan plan) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // 16-byte chunk
  const int per_bh = kHeadDim * 2 / 16;
  const int n_bh = batch * heads;
  if (i >= 2 * n_bh * per_bh) return;
  const int tensor = i / (n_bh * per_bh);
  const int r = i % (n_bh * per_bh);
  const int bh = r / per_bh, ch = r % per_bh;
  const int pos = plan.pos[bh / heads];
  if (pos < 0) return;
  const uint4* src = reinterpret_cast<const uint4*>((tensor ? v : k) + (size_t)bh * kHeadDim);
  uint4* dst = reinterpret_cast<uint4*>((tensor ? v_tail : k_tail) + ((size_t)bh * kBlockTokens + pos) * kHeadDim);
  dst[ch] = src[ch];
}

// Zeroes the index entries a call will publish (the look-back reads 0 as "not yet
// published"), wherever the plan and the block table put them.
template <class Plan>
__global__ void clear_entries_kernel(const EncodeArgs a, const __grid_constant__ Plan plan, long n_call) {
  const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_call) return;
  const size_t e = call_block(a, plan, t).entry;
  reinterpret_cast<unsigned long long*>(a.k_index)[e] = 0ull;
  reinterpret_cast<unsigned long long*>(a.v_index)[e] = 0ull;
}

template <class Plan>
cudaError_t launch_encode_t(const EncodeArgs& a, const Plan& plan, cudaStream_t stream) {
  const size_t smem = sizeof(EncodeSmem);
  static bool configured = false;  // per process; the attribute is per function, not per device
  if (!configured) {
    const cudaError_t e = cudaFuncSetAttribute(encode_kernel<Plan>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const long n_call = (long)a.batch * a.heads * a.nb;
  // the look-back reads the new index entries as "not yet published" (0), and the
  // ticket and done counters start from zero
  cudaError_t e = cudaSuccess;
  if (!a.ragged && a.block_table == nullptr) {
    const size_t pitch = (size_t)a.max_blocks * 8;
    const size_t width = (size_t)a.nb * 8;
    const size_t height = (size_t)a.batch * a.heads;
    e = cudaMemset2DAsync(a.k_index + (size_t)a.n_old * 2, pitch, 0, width, height, stream);
    if (e == cudaSuccess) e = cudaMemset2DAsync(a.v_index + (size_t)a.n_old * 2, pitch, 0, width, height, stream);
  } else {
    clear_entries_kernel<Plan><<<(unsigned)((n_call + 255) / 256), 256, 0, stream>>>(a, plan, n_call);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(a.ctrl + kCtrlScratch, 0, sizeof(uint64_t), stream);
  if (e != cudaSuccess) return e;
  encode_kernel<Plan><<<(unsigned)n_call, kEncodeThreads, smem, stream>>>(a, plan);
  return cudaGetLastError();
}

struct NoEncodePlan {};

}  // namespace

size_t encode_smem_bytes() { return sizeof(EncodeSmem); }

cudaError_t launch_encode(const EncodeArgs& a, const RaggedEncodePlan* plan, cudaStream_t stream) {
  if (a.ragged) return launch_encode_t<RaggedEncodePlan>(a, *plan, stream);
  return launch_encode_t<NoEncodePlan>(a, NoEncodePlan{}, stream);
}

cudaError_t launch_append(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail, int n_bh,
                          int pos, cudaStream_t stream) {
  const int chunks = 2 * n_bh * (kHeadDim * 2 / 16);
  append_tail_kernel<<<(chunks + 255) / 256, 256, 0, stream>>>(k, v, k_tail, v_tail, n_bh, pos);
  return cudaGetLastError();
}

cudaError_t launch_append_ragged(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail,
                                 int batch, int heads, const RaggedAppendPlan& plan, cudaStream_t stream) {
  const int chunks = 2 * batch * heads * (kHeadDim * 2 / 16);
  append_tail_ragged_kernel<<<(chunks + 255) / 256, 256, 0, stream>>>(k, v, k_tail, v_tail, batch, heads, plan);
  return cudaGetLastError();
}

}  // namespace packkv
