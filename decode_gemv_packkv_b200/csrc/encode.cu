// PackKV encoder: block quantization, joint token reorder, channel-direction
// bit-packing (FORMAT.md sections 1-4; PackKV paper page, Figure 2 steps (1)
// and (2), Figure 5 granularities, TL;DR).
//
// One encode call runs three kernels on the caller's stream:
//   1. encode_kernel<false>: per (sequence, head, block) CTA, quantize + reorder
//      + unit widths, and store the record length in the index;
//   2. arena_scan_kernel: one CTA turns the lengths into arena offsets in
//      ascending (sequence, head, block) order, advances the arena ends and
//      checks capacity (so the arena layout is deterministic);
//   3. encode_kernel<true>: recomputes the block (cheaper than staging the codes
//      in a workspace the ABI does not have), assembles the record in shared
//      memory and writes it with 16-byte stores at its offset.
// The encoder runs once per 128 tokens per head; it is not on the per-token path.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace packkv {

struct EncodeSmem {
  __half kx[kBlockTokens][kHeadDim];   // input K block; later the K record buffer
  __half vx[kBlockTokens][kHeadDim];   // input V block; later the V record buffer
  uint8_t ck[kBlockTokens][kHeadDim];  // K codes [token][channel]
  uint8_t cv[kBlockTokens][kHeadDim];  // V codes [token][channel]
  uint16_t kmin[kHeadDim], kscale[kHeadDim];     // per channel
  uint16_t vmin[kBlockTokens], vscale[kBlockTokens];  // per token (original order)
  int key[kBlockTokens];
  uint8_t perm[kBlockTokens];          // perm[slot] = token
  uint8_t base[2][kGroups][kHeadDim];
  uint8_t width[2][kGroups][kHeadDim];
  uint16_t ustart[2][kGroups][kHeadDim];  // word index of each unit in the word area
  int group_total[2][kGroups];
  int wsum[2];
  int nonfinite;
};

__device__ __forceinline__ int bitlen(uint32_t x) { return x == 0 ? 0 : 32 - __clz(x); }

template <bool kWrite>
__global__ void __launch_bounds__(256) encode_kernel(EncodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EncodeSmem& s = *reinterpret_cast<EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int blk = blockIdx.x % a.nb;
  const int bh = blockIdx.x / a.nb;  // b * heads + h
  const int qmax = (1 << a.bits) - 1;
  const size_t in_base = ((size_t)bh * a.nb + blk) * kBlockTokens * kHeadDim;
  const size_t slot = (size_t)bh * a.max_blocks + a.n_old + blk;

  if (kWrite) {
    // the scan kernel marks a whole call as failed when an arena would overflow
    const uint64_t fail = a.ctrl[kCtrlScratch];
    if (fail) return;
  }

  // ---- load both blocks (16-byte vectors), flag non-finite values ----------
  if (tid == 0) s.nonfinite = 0;
  if (tid < 2) s.wsum[tid] = 0;
  __syncthreads();
  {
    const uint4* ksrc = reinterpret_cast<const uint4*>(a.k + in_base);
    const uint4* vsrc = reinterpret_cast<const uint4*>(a.v + in_base);
    uint4* kdst = reinterpret_cast<uint4*>(&s.kx[0][0]);
    uint4* vdst = reinterpret_cast<uint4*>(&s.vx[0][0]);
    int bad = 0;
    for (int i = tid; i < kBlockTokens * kHeadDim / 8; i += blockDim.x) {
      uint4 kk = ksrc[i], vv = vsrc[i];
      kdst[i] = kk;
      vdst[i] = vv;
      const uint32_t w[8] = {kk.x, kk.y, kk.z, kk.w, vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        bad |= ((w[j] & 0x7C00u) == 0x7C00u) | ((w[j] & 0x7C000000u) == 0x7C000000u);
      }
    }
    if (bad) s.nonfinite = 1;
  }
  __syncthreads();
  if (!kWrite && tid == 0 && s.nonfinite) set_status(a.ctrl, PACKKV_DEV_NONFINITE);

  // ---- quantization parameters: K per channel, V per token -----------------
  {
    float mn = 3.4e38f, mx = -3.4e38f;
    if (tid < kHeadDim) {
      const int c = tid;
      for (int t = 0; t < kBlockTokens; ++t) {
        const float x = __half2float(s.kx[t][c]);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
    } else {
      const int t = tid - kHeadDim;
      for (int i = 0; i < kHeadDim; ++i) {
        const float x = __half2float(s.vx[t][(i + t) & (kHeadDim - 1)]);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
    }
    if (mn == 0.0f) mn = 0.0f;  // -0 is stored as +0
    const float range = __fsub_rn(mx, mn);
    uint16_t sc = 0;
    if (range > 0.0f) sc = __half_as_ushort(__float2half_ru(__fdiv_rn(range, (float)qmax)));
    const uint16_t mnb = __half_as_ushort(__float2half_rn(mn));  // exact: mn is an fp16 value
    if (tid < kHeadDim) {
      s.kmin[tid] = mnb;
      s.kscale[tid] = sc;
    } else {
      s.vmin[tid - kHeadDim] = mnb;
      s.vscale[tid - kHeadDim] = sc;
    }
  }
  __syncthreads();

  // ---- codes -----------------------------------------------------------------
  for (int e = tid; e < kBlockTokens * kHeadDim; e += blockDim.x) {
    const int t = e >> 7, c = e & 127;
    {
      const float sc = half_bits_to_float(s.kscale[c]);
      int code = 0;
      if (sc > 0.0f) {
        const float y = __fdiv_rn(__fsub_rn(__half2float(s.kx[t][c]), half_bits_to_float(s.kmin[c])), sc);
        code = (int)fminf(fmaxf(rintf(y), 0.0f), (float)qmax);
      }
      s.ck[t][c] = (uint8_t)code;
    }
    {
      const float sc = half_bits_to_float(s.vscale[t]);
      int code = 0;
      if (sc > 0.0f) {
        const float y = __fdiv_rn(__fsub_rn(__half2float(s.vx[t][c]), half_bits_to_float(s.vmin[t])), sc);
        code = (int)fminf(fmaxf(rintf(y), 0.0f), (float)qmax);
      }
      s.cv[t][c] = (uint8_t)code;
    }
  }
  __syncthreads();

  // ---- reorder key per token, then stable rank ------------------------------
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < kBlockTokens; t += blockDim.x / 32) {
      uint32_t sum = 0;
      if (a.key_kind != PACKKV_KEY_IDENTITY) {
        sum = __dp4a(reinterpret_cast<const uint32_t*>(s.ck[t])[lane], 0x01010101u, 0u);
        if (a.key_kind == PACKKV_KEY_KV_SUM)
          sum = __dp4a(reinterpret_cast<const uint32_t*>(s.cv[t])[lane], 0x01010101u, sum);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) s.key[t] = (int)sum;
    }
  }
  __syncthreads();
  if (tid < kBlockTokens) {
    const int kt = s.key[tid];
    int r = 0;
    for (int u = 0; u < kBlockTokens; ++u) {
      const int ku = s.key[u];
      r += (ku < kt) | ((ku == kt) & (u < tid));
    }
    s.perm[r] = (uint8_t)tid;
  }
  __syncthreads();

  // ---- frame of reference and width of every (group, channel) unit ----------
  for (int u = tid; u < 2 * kGroups * kHeadDim; u += blockDim.x) {
    const int tensor = u >> 9, g = (u >> 7) & 3, c = u & 127;
    const uint8_t(*cx)[kHeadDim] = tensor ? s.cv : s.ck;
    int lo = 255, hi = 0;
    for (int j = 0; j < kGroupTokens; ++j) {
      const int code = cx[s.perm[g * kGroupTokens + j]][c];
      lo = min(lo, code);
      hi = max(hi, code);
    }
    s.base[tensor][g][c] = (uint8_t)lo;
    s.width[tensor][g][c] = (uint8_t)bitlen((uint32_t)(hi - lo));
    atomicAdd(&s.wsum[tensor], bitlen((uint32_t)(hi - lo)));
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

  if (!kWrite) {
    if (tid == 0) {
      a.k_index[slot * 2 + 1] = (uint32_t)(rec_bytes[0] >> 4);
      a.v_index[slot * 2 + 1] = (uint32_t)(rec_bytes[1] >> 4);
    }
    return;
  }

  // ---- write pass: unit word offsets ----------------------------------------
  {
    const int warp = tid >> 5, lane = tid & 31;  // 8 warps = (tensor, group)
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

  // ---- assemble both records in shared memory (reusing the input buffers) ---
  uint32_t* rec32[2] = {reinterpret_cast<uint32_t*>(&s.kx[0][0]), reinterpret_cast<uint32_t*>(&s.vx[0][0])};
  for (int i = tid; i < raw_bytes / 4; i += blockDim.x) {
    rec32[0][i] = 0u;
    rec32[1][i] = 0u;
  }
  __syncthreads();
#pragma unroll
  for (int tensor = 0; tensor < 2; ++tensor) {
    unsigned char* rec = reinterpret_cast<unsigned char*>(rec32[tensor]);
    if (tid == 0) {
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
    }
    if (tid < kHeadDim) {
      uint16_t* mn = reinterpret_cast<uint16_t*>(rec + kParamOffset);
      uint16_t* sc = mn + kHeadDim;
      if (tensor == 0) {
        mn[tid] = s.kmin[tid];
        sc[tid] = s.kscale[tid];
      } else {
        mn[tid] = s.vmin[s.perm[tid]];
        sc[tid] = s.vscale[s.perm[tid]];
      }
    }
    if (!raw[tensor]) {
      for (int u = tid; u < kGroups * kHeadDim; u += blockDim.x) {
        const int g = u >> 7, c = u & 127;
        rec[kMetaOffset + u] = (uint8_t)(s.base[tensor][g][c] | (s.width[tensor][g][c] << 4));
      }
    }
  }
  // raw records of b = 2 / 4: words in 8-bit tensor-core fragment order (FORMAT.md section 4).
  // A[m][k] = code of slot m, channel k (K) or of slot k, channel m (V).
  if (a.bits != 3) {
#pragma unroll
    for (int tensor = 0; tensor < 2; ++tensor) {
      if (!raw[tensor]) continue;
      uint32_t* words = rec32[tensor] + kRawWordOffset / 4;
      for (int wi = tid; wi < 512 * a.bits; wi += blockDim.x) {
        // wi = ((tile row or tile pair)*2 + J)*32 + lane)*4 + 2*Q2 + kh, kappa = 2J + Q2
        const int kh = wi & 1, q2 = (wi >> 1) & 1, lane = (wi >> 2) & 31, jj = (wi >> 7) & 1, tp = wi >> 8;
        const int kappa = 2 * jj + q2, g = lane >> 2, t = lane & 3;
        uint32_t word = 0;
        const int nfields = 32 / a.bits;
        for (int f = 0; f < nfields; ++f) {
          int e, rh, tile;
          if (a.bits == 4) {
            e = f >> 1, rh = f & 1, tile = tp;
          } else {
            e = f >> 2, rh = f & 1, tile = 2 * tp + ((f >> 1) & 1);
          }
          const int m = 16 * tile + 8 * rh + g, k = 32 * kappa + 16 * kh + 4 * t + e;
          const uint32_t code = tensor ? s.cv[s.perm[k]][m] : s.ck[s.perm[m]][k];
          word |= code << (a.bits * f);
        }
        words[wi] = word;
      }
    }
  }
  // pack the units: every word is owned by exactly one thread
  for (int u = tid; u < 2 * kGroups * kHeadDim; u += blockDim.x) {
    const int tensor = u >> 9, g = (u >> 7) & 3, c = u & 127;
    if (raw[tensor] && a.bits != 3) continue;  // written above
    const uint8_t(*cx)[kHeadDim] = tensor ? s.cv : s.ck;
    const int w = raw[tensor] ? a.bits : s.width[tensor][g][c];
    const int base = raw[tensor] ? 0 : s.base[tensor][g][c];
    if (w == 0) continue;
    int gstart = 0;
    for (int gg = 0; gg < g; ++gg) gstart += s.group_total[tensor][gg];
    uint32_t* words = rec32[tensor] + (raw[tensor] ? kRawWordOffset : kPackedWordOffset) / 4 + gstart +
                      s.ustart[tensor][g][c];
    // slices in descending size: 4 | 2 then 1 | 2 | 1
    int lo = 0, at = 0;
    int rem = w;
    while (rem > 0) {
      const int p = rem >= 4 ? 4 : (rem >= 2 ? 2 : 1);
      const uint32_t mask = (1u << p) - 1u;
      for (int q = 0; q < p; ++q) {
        uint32_t word = 0;
        const int per = 32 / p;
        for (int f = 0; f < per; ++f) {
          const int j = q * per + f;
          const uint32_t off = (uint32_t)(cx[s.perm[g * kGroupTokens + j]][c] - base);
          word |= ((off >> lo) & mask) << ((j * p) & 31);
        }
        words[at + q] = word;
      }
      at += p;
      lo += p;
      rem -= p;
    }
  }
  __syncthreads();

  // ---- write the records and the permutation --------------------------------
#pragma unroll
  for (int tensor = 0; tensor < 2; ++tensor) {
    const uint32_t* index = tensor ? a.v_index : a.k_index;
    uint8_t* arena = tensor ? a.v_arena : a.k_arena;
    const uint64_t off16 = index[slot * 2];
    uint4* dst = reinterpret_cast<uint4*>(arena + off16 * 16);
    const uint4* src = reinterpret_cast<const uint4*>(rec32[tensor]);
    for (int i = tid; i < rec_bytes[tensor] / 16; i += blockDim.x) dst[i] = src[i];
  }
  if (a.perm != nullptr && tid < kBlockTokens) a.perm[slot * kBlockTokens + tid] = s.perm[tid];
}

// One CTA: arena offsets from record lengths, in (sequence, head, block) order.
__global__ void __launch_bounds__(1024) arena_scan_kernel(EncodeArgs a) {
  __shared__ unsigned long long warp_sums[32];
  __shared__ unsigned long long totals[2];
  __shared__ int failed;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long n = (long)a.batch * a.heads * a.nb;
  const long per = (n + blockDim.x - 1) / blockDim.x;
  const long first = min(n, per * tid), last = min(n, first + per);
  if (tid == 0) failed = 0;
  for (int tensor = 0; tensor < 2; ++tensor) {
    uint32_t* index = tensor ? a.v_index : a.k_index;
    auto entry = [&](long e) -> uint32_t* {
      const long bh = e / a.nb, i = e % a.nb;
      return index + ((size_t)bh * a.max_blocks + a.n_old + i) * 2;
    };
    unsigned long long local = 0;
    for (long e = first; e < last; ++e) local += entry(e)[1];
    unsigned long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      unsigned long long ws = warp_sums[lane];
      unsigned long long wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      warp_sums[lane] = wi - ws;
      if (lane == 31) totals[tensor] = wi;
    }
    __syncthreads();
    const unsigned long long end = a.ctrl[tensor ? kCtrlVEnd : kCtrlKEnd];
    const unsigned long long total = totals[tensor];
    const bool fits = (end + total) * 16ull <= a.arena_bytes;
    if (!fits && tid == 0) failed = 1;
    unsigned long long at = end + warp_sums[warp] + (incl - local);
    for (long e = first; e < last; ++e) {
      uint32_t* ent = entry(e);
      const uint32_t len = ent[1];
      ent[0] = fits ? (uint32_t)at : 0xFFFFFFFFu;
      if (!fits) ent[1] = 0u;
      at += len;
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (failed) {
      // neither arena advances; the write pass skips the whole call
      a.ctrl[kCtrlScratch] = 1ull;
      set_status(a.ctrl, PACKKV_DEV_CAPACITY);
    } else {
      a.ctrl[kCtrlScratch] = 0ull;
      a.ctrl[kCtrlKEnd] += totals[0];
      a.ctrl[kCtrlVEnd] += totals[1];
    }
  }
  if (failed) {
    // mark every new entry of both tensors invalid (the K pass above may have fit)
    for (int tensor = 0; tensor < 2; ++tensor) {
      uint32_t* index = tensor ? a.v_index : a.k_index;
      for (long e = first; e < last; ++e) {
        const long bh = e / a.nb, i = e % a.nb;
        uint32_t* ent = index + ((size_t)bh * a.max_blocks + a.n_old + i) * 2;
        ent[0] = 0xFFFFFFFFu;
        ent[1] = 0u;
      }
    }
  }
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

size_t encode_smem_bytes() { return sizeof(EncodeSmem); }

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(EncodeSmem);
  static bool configured = false;  // per process; the attribute is per function, not per device
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(encode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const unsigned grid = (unsigned)((long)a.batch * a.heads * a.nb);
  encode_kernel<false><<<grid, 256, smem, stream>>>(a);
  arena_scan_kernel<<<1, 1024, 0, stream>>>(a);
  encode_kernel<true><<<grid, 256, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const uint16_t* k, const uint16_t* v, uint16_t* k_tail, uint16_t* v_tail, int n_bh,
                          int pos, cudaStream_t stream) {
  const int chunks = 2 * n_bh * (kHeadDim * 2 / 16);
  append_tail_kernel<<<(chunks + 255) / 256, 256, 0, stream>>>(k, v, k_tail, v_tail, n_bh, pos);
  return cudaGetLastError();
}

}  // namespace packkv
