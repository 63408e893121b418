"""CPU oracle for the PackKV packed KV cache and its two decode GEMVs.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
shares no code, tables or constants with the CUDA library; both follow the
written packed-cache format (version 1) independently.

Sources (the PackKV pages; cited by page title and figure/section):
  [Abs]    "PackKV: Reducing KV Cache Memory Footprint through LLM-Aware Lossy
           Compression", abstract: dynamic growth of the cache, fused
           decompression + matrix-vector product.
  [TLDR]   same page, TL;DR: quantization + light lossless encoding; reorder
           exploiting attention's permutation invariance with K/V bound together;
           decompression inside the matrix-vector product.
  [Fig. 1] attention at decode: q dots every K, softmax, weighted sum of V.
  [Fig. 2] step (1) reorder the quantized vectors, step (2) bit-pack the integer
           codes in the channel direction.
  [Fig. 5] token-wise vs channel-wise quantization granularity.
  [Viz]    "PackKV Lossy Compression for KV Caches" visualisation page,
           section "Permutation invariance, visually".

The pages fix none of the numbers; the readings taken (block 128, group 32,
K per channel / V per token, min-max quantizer with an fp16 scale rounded up,
K-code-sum reorder key, frame-of-reference + width packing in power-of-two
slices) are the ones the packed-cache format v1 fixes.

Floating point: the quantizer is defined in fp32 (single IEEE operations, as the
GPU performs them) so that integer codes agree bit for bit; decoding and both
products are fp64.  Every function is pinned by tests in tests/test_oracle_*.py
against values fixed by hand from the format, by brute force or by closed forms.
"""
from __future__ import annotations

import struct
from dataclasses import dataclass, field

import numpy as np

BLOCK_TOKENS = 128
GROUP_TOKENS = 32
HEAD_DIM = 128
GROUPS_PER_BLOCK = BLOCK_TOKENS // GROUP_TOKENS
FORMAT_VERSION = 1
RAW_FLAG = 0x1
V_FLAG = 0x2

KEY_IDENTITY = 0
KEY_K_SUM = 1
KEY_KV_SUM = 2

FP16_MAX = 65504.0


# ----------------------------------------------------------------------------
# fp16 rounding toward +infinity, from the IEEE-754 binary16 definition
# ----------------------------------------------------------------------------
def fp16_round_up(x32: np.ndarray) -> np.ndarray:
    """Smallest binary16 value >= x, for finite x >= 0 (array of float32).

    binary16 has 10 fraction bits, exponent range [-14, 15] and subnormals with
    spacing 2^-24.  In the binade [2^e, 2^(e+1)) (e >= -14) the spacing is
    2^(e-10); below 2^-14 it is 2^-24.  The result is ceil(x / spacing) * spacing,
    computed exactly in fp64 (x / spacing is an exact power-of-two scaling).
    Values above 65504 round up to +inf.
    """
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError("fp16_round_up is defined here for finite x >= 0")
    out = np.zeros(x.shape, dtype=np.float64)
    pos = x > 0
    xp = x[pos]
    _, e_plus_1 = np.frexp(xp)            # xp = m * 2^E, m in [0.5, 1)  ->  floor(log2 xp) = E - 1
    e = e_plus_1.astype(np.int64) - 1
    e = np.maximum(e, -14)                # subnormal range shares the 2^-24 spacing
    spacing = np.ldexp(1.0, (e - 10).astype(np.int32))
    out[pos] = np.ceil(xp / spacing) * spacing
    out[out > FP16_MAX] = np.inf
    return out.astype(np.float16)       # exact: every value is on the binary16 grid


# ----------------------------------------------------------------------------
# Step 1: block quantization ([Fig. 5] granularities; [Fig. 2], [TLDR] "quantize")
# ----------------------------------------------------------------------------
def quantize_rows(x16: np.ndarray, bits: int):
    """Asymmetric min/max quantization of each row (last axis) of an fp16 array.

    Returns (codes uint8 like x16, mn fp16 [rows], scale fp16 [rows]):
      mn = min(row) (exact; -0 stored as +0), range = f32(max) - f32(mn),
      scale = fp16_round_up(range / (2^b - 1)), or 0 when range == 0;
      code = clamp(rint((f32(x) - f32(mn)) / f32(scale)), 0, 2^b - 1), rint half-even.
    """
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    x16 = np.asarray(x16, dtype=np.float16)
    if not np.all(np.isfinite(x16)):
        raise ValueError("quantizer input must be finite")
    qmax = (1 << bits) - 1
    mn = x16.min(axis=-1)
    mx = x16.max(axis=-1)
    mn = np.where(mn == 0, np.float16(0.0), mn).astype(np.float16)
    rng = mx.astype(np.float32) - mn.astype(np.float32)          # fp32 RN
    s = rng / np.float32(qmax)                                   # fp32 RN
    live = rng > 0
    scale = np.zeros(mn.shape, dtype=np.float16)
    scale[live] = fp16_round_up(s[live])
    x32 = x16.astype(np.float32)
    diff = x32 - mn.astype(np.float32)[..., None]                # fp32 RN
    safe = np.where(live, scale.astype(np.float32), np.float32(1.0))
    y = diff / safe[..., None]                                   # fp32 RN
    codes = np.clip(np.rint(y), 0, qmax)                         # half-even
    codes = np.where(live[..., None], codes, 0).astype(np.uint8)
    return codes, mn, scale


def quantize_block_k(k_blk: np.ndarray, bits: int):
    """K block [128 tokens, 128 channels] -> codes [t, c], per-channel mn/scale [c]."""
    codes_ct, mn, sc = quantize_rows(np.asarray(k_blk, np.float16).T, bits)
    return codes_ct.T.copy(), mn, sc


def quantize_block_v(v_blk: np.ndarray, bits: int):
    """V block [128 tokens, 128 channels] -> codes [t, c], per-token mn/scale [t]."""
    return quantize_rows(np.asarray(v_blk, np.float16), bits)


def quant_error_bound(scale16: np.ndarray, bits: int) -> np.ndarray:
    """Per-element bound on |x - x_hat| for the quantizer above.

    With d = x - mn >= 0 and S = scale: fl(d) = d(1+e1), y = fl(fl(d)/S) =
    (fl(d)/S)(1+e2), |e1|,|e2| <= 2^-24.  rint moves y by at most 1/2 and never
    needs the clamp (y < 2^b - 1/2 because S >= s >= range(1-2^-24)^2/(2^b-1)).
    So |d - S*code| <= S*|d/S - y| + S/2 <= S*(2^b-1)(1+2^-23)(2^-23+2^-48) + S/2
    < S*(1/2 + 2^(b-23)) <= S*(1/2 + 2^(b-22)).
    """
    return np.asarray(scale16, np.float64) * (0.5 + 2.0 ** (bits - 22))


# ----------------------------------------------------------------------------
# Step 2: joint token reorder ([Fig. 2] step 1; [TLDR]; [Viz] permutation invariance)
# ----------------------------------------------------------------------------
def reorder_keys(codes_k: np.ndarray, codes_v: np.ndarray, key_kind: int) -> np.ndarray:
    """Integer sort key per token: 0 identity, 1 sum of K codes, 2 sum of K and V codes."""
    n = codes_k.shape[0]
    if key_kind == KEY_IDENTITY:
        return np.zeros(n, dtype=np.int64)
    if key_kind == KEY_K_SUM:
        return codes_k.astype(np.int64).sum(axis=1)
    if key_kind == KEY_KV_SUM:
        return codes_k.astype(np.int64).sum(axis=1) + codes_v.astype(np.int64).sum(axis=1)
    raise ValueError("unknown reorder key")


def stable_rank(keys: np.ndarray) -> np.ndarray:
    """rank[t] = #{u : key[u] < key[t] or (key[u] == key[t] and u < t)}."""
    keys = np.asarray(keys, dtype=np.int64)
    t = np.arange(keys.shape[0])
    less = keys[None, :] < keys[:, None]
    tie_before = (keys[None, :] == keys[:, None]) & (t[None, :] < t[:, None])
    return (less | tie_before).sum(axis=1).astype(np.int64)


# ----------------------------------------------------------------------------
# Step 3: bit-packing along a channel ([Fig. 2] step 2; [TLDR] light lossless encoding)
# ----------------------------------------------------------------------------
def slices_of_width(w: int):
    """Power-of-two slices (p bits starting at offset bit lo), largest first."""
    return {0: [], 1: [(1, 0)], 2: [(2, 0)], 3: [(2, 0), (1, 2)], 4: [(4, 0)]}[w]


UNITS_FOR = 0          # frame of reference: base = min of the unit's codes (format v1 default)
UNITS_WIDTH_ONLY = 1   # no base: base = 0, the width covers the largest code ([Fig. 3] ablation)


def unit_base_width(codes32: np.ndarray, unit_mode: int = UNITS_FOR):
    """Base and width of one (group, channel) unit: frame of reference (base = min,
    w = bitlen(max - min)) or, width-only, base = 0 and w = bitlen(max).  Both are
    format v1 units: the record stores base | w << 4 either way."""
    c = np.asarray(codes32, dtype=np.int64)
    base = int(c.min()) if unit_mode == UNITS_FOR else 0
    w = int(c.max() - base).bit_length()
    return base, w


def pack_unit(offsets32: np.ndarray, w: int) -> np.ndarray:
    """Pack 32 offsets (each < 2^w) into w uint32 words, slice by slice."""
    offs = np.asarray(offsets32, dtype=np.uint64)
    assert offs.shape == (GROUP_TOKENS,)
    assert w == 0 or int(offs.max()) < (1 << w)
    words = []
    j = np.arange(GROUP_TOKENS, dtype=np.uint64)
    for p, lo in slices_of_width(w):
        fields = (offs >> np.uint64(lo)) & np.uint64((1 << p) - 1)
        bitpos = j * np.uint64(p)
        slice_words = np.zeros(p, dtype=np.uint64)
        np.bitwise_or.at(slice_words, (bitpos // np.uint64(32)).astype(np.int64),
                         fields << (bitpos % np.uint64(32)))
        words.append(slice_words)
    if not words:
        return np.zeros(0, dtype=np.uint32)
    return np.concatenate(words).astype(np.uint32)


def unpack_unit(words: np.ndarray, w: int) -> np.ndarray:
    """Inverse of pack_unit: w words -> 32 offsets."""
    words = np.asarray(words, dtype=np.uint64)
    assert words.shape == (w,)
    offs = np.zeros(GROUP_TOKENS, dtype=np.uint64)
    j = np.arange(GROUP_TOKENS, dtype=np.uint64)
    at = 0
    for p, lo in slices_of_width(w):
        sl = words[at:at + p]
        at += p
        bitpos = j * np.uint64(p)
        fields = (sl[(bitpos // np.uint64(32)).astype(np.int64)] >> (bitpos % np.uint64(32))) \
            & np.uint64((1 << p) - 1)
        offs |= fields << np.uint64(lo)
    return offs.astype(np.int64)


# ----------------------------------------------------------------------------
# Step 4: record assembly (packed-cache format v1, section 4)
# ----------------------------------------------------------------------------
def raw_record_bytes(bits: int) -> int:
    return 16 + 512 + 2048 * bits


def record_bytes_max(bits: int) -> int:
    """A compressed record is always strictly smaller than the raw one."""
    return raw_record_bytes(bits)


def frag_word_bit(bits: int, m: int, k: int):
    """(word index, bit offset) of A[m][k] in the raw fragment order (b = 2, 4).

    Restates packed-cache format v1, section 4: m = 16T + 8rh + g, k = 32kappa + 16kh + 4t + e,
    lane = 4g + t; the word is picked by (row tile T (b = 4) or tile pair T div 2
    (b = 2), kappa, kh, lane) and the field inside it by (e, rh) (and the tile
    row parity for b = 2): byte e of the word holds row g in its low field(s)
    and row g + 8 above them.
    """
    T, rh, g = m // 16, (m // 8) % 2, m % 8
    kappa, kh, t, e = k // 32, (k // 16) % 2, (k % 16) // 4, k % 4
    lane = 4 * g + t
    J, Q2 = kappa // 2, kappa % 2
    if bits == 4:
        return ((T * 2 + J) * 32 + lane) * 4 + 2 * Q2 + kh, 4 * (2 * e + rh)
    if bits == 2:
        return (((T // 2) * 2 + J) * 32 + lane) * 4 + 2 * Q2 + kh, 2 * (4 * e + 2 * (T % 2) + rh)
    raise ValueError("fragment order is defined for b = 2 and b = 4")


def frag_plane_bit(m: int, k: int):
    """(word index within the 1-bit plane, bit offset) of A[m][k]'s high bit in a raw
    b = 3 record (packed-cache format v1, section 4): the word is picked by (tile quad T div 4,
    kappa, kh, lane), the bit by (e, T mod 4, rh)."""
    T, rh, g = m // 16, (m // 8) % 2, m % 8
    kappa, kh, t, e = k // 32, (k // 16) % 2, (k % 16) // 4, k % 4
    lane = 4 * g + t
    J, Q2 = kappa // 2, kappa % 2
    return (((T // 4) * 2 + J) * 32 + lane) * 4 + 2 * Q2 + kh, 8 * e + 2 * (T % 4) + rh


def frag_fields(bits: int, m: int, k: int):
    """Where the bits of A[m][k] live in a raw record's word area: a list of
    (word, bit offset, field width, code bit offset).  b = 2 / 4: one field of b
    bits.  b = 3: bits 0-1 in the 2-bit plane (words 0 .. 1023, the b = 2 order),
    bit 2 in the 1-bit plane (words 1024 .. 1535)."""
    if bits in (2, 4):
        w, bit = frag_word_bit(bits, m, k)
        return [(w, bit, bits, 0)]
    if bits == 3:
        w0, b0 = frag_word_bit(2, m, k)
        w1, b1 = frag_plane_bit(m, k)
        return [(w0, b0, 2, 0), (1024 + w1, b1, 1, 2)]
    raise ValueError("raw records hold 2, 3 or 4-bit codes")


def pack_raw_fragment(a: np.ndarray, bits: int) -> np.ndarray:
    """Raw word area of a record: every code of the 128x128 matrix A at its place(s)."""
    words = [0] * (512 * bits)
    for m in range(128):
        for k in range(128):
            code = int(a[m, k])
            for w, bit, width, shift in frag_fields(bits, m, k):
                words[w] |= ((code >> shift) & ((1 << width) - 1)) << bit
    return np.array(words, dtype=np.uint64).astype(np.uint32)


def unpack_raw_fragment(words: np.ndarray, bits: int) -> np.ndarray:
    a = np.zeros((128, 128), np.int64)
    for m in range(128):
        for k in range(128):
            code = 0
            for w, bit, width, shift in frag_fields(bits, m, k):
                code |= ((int(words[w]) >> bit) & ((1 << width) - 1)) << shift
            a[m, k] = code
    return a


def _ceil16(n: int) -> int:
    return (n + 15) // 16 * 16


def build_record(codes_slot: np.ndarray, mn16: np.ndarray, sc16: np.ndarray,
                 bits: int, is_v: bool, unit_mode: int = UNITS_FOR) -> bytes:
    """Assemble one record from codes in storage order [slot, channel] and params
    (units sized by unit_base_width in `unit_mode`)."""
    codes_slot = np.asarray(codes_slot, dtype=np.int64)
    assert codes_slot.shape == (BLOCK_TOKENS, HEAD_DIM)
    base = np.zeros((GROUPS_PER_BLOCK, HEAD_DIM), dtype=np.int64)
    width = np.zeros((GROUPS_PER_BLOCK, HEAD_DIM), dtype=np.int64)
    for g in range(GROUPS_PER_BLOCK):
        for c in range(HEAD_DIM):
            base[g, c], width[g, c] = unit_base_width(codes_slot[32 * g:32 * g + 32, c], unit_mode)
    compressed_size = _ceil16(1040 + 4 * int(width.sum()))
    raw = compressed_size >= raw_record_bytes(bits)
    if raw:
        base[:] = 0
        width[:] = bits
    words = []
    group_start = []
    for g in range(GROUPS_PER_BLOCK):
        group_start.append(sum(len(w_) for w_ in words))
        for c in range(HEAD_DIM):
            offs = codes_slot[32 * g:32 * g + 32, c] - base[g, c]
            words.append(pack_unit(offs, int(width[g, c])))
    all_words = np.concatenate(words).astype(np.uint32) if words else np.zeros(0, np.uint32)
    if raw:
        # same header values, word area in tensor-core fragment order (K: rows = slots, V: rows = channels)
        all_words = pack_raw_fragment(codes_slot.T if is_v else codes_slot, bits)
    flags = (RAW_FLAG if raw else 0) | (V_FLAG if is_v else 0) | (FORMAT_VERSION << 8) | (bits << 16)
    out = bytearray()
    out += struct.pack("<4H", *group_start)
    out += struct.pack("<II", flags, int(all_words.size))
    out += np.asarray(mn16, dtype=np.float16).tobytes()
    out += np.asarray(sc16, dtype=np.float16).tobytes()
    if not raw:
        out += (base | (width << 4)).astype(np.uint8).tobytes()
    out += all_words.astype("<u4").tobytes()
    out += b"\x00" * (_ceil16(len(out)) - len(out))
    assert len(out) <= record_bytes_max(bits)
    assert raw == (len(out) == raw_record_bytes(bits))
    return bytes(out)


@dataclass
class ParsedRecord:
    raw: bool
    is_v: bool
    bits: int
    mn: np.ndarray          # fp16 [128]
    scale: np.ndarray       # fp16 [128]
    base: np.ndarray        # int [4, 128]
    width: np.ndarray       # int [4, 128]
    codes: np.ndarray       # int [slot, channel]
    group_word_start: list = field(default_factory=list)


def parse_record(rec: bytes) -> ParsedRecord:
    """Decode one record back to codes and parameters (inverse of build_record)."""
    gws = list(struct.unpack_from("<4H", rec, 0))
    flags, total_words = struct.unpack_from("<II", rec, 8)
    raw = bool(flags & RAW_FLAG)
    is_v = bool(flags & V_FLAG)
    version = (flags >> 8) & 0xFF
    bits = (flags >> 16) & 0xF
    if version != FORMAT_VERSION:
        raise ValueError("unknown record version")
    if flags >> 24:
        raise ValueError("a layout-variant record (parse_record_variant reads those)")
    mn = np.frombuffer(rec, dtype="<f2", count=128, offset=16).astype(np.float16)
    sc = np.frombuffer(rec, dtype="<f2", count=128, offset=272).astype(np.float16)
    if raw:
        # a raw record keeps the header values of the unit layout with every width = b
        if gws != [g * 128 * bits for g in range(4)] or total_words != 512 * bits:
            raise ValueError("raw record header does not match the unit layout")
        base = np.zeros((4, 128), np.int64)
        width = np.full((4, 128), bits, np.int64)
        word_at = 528
    else:
        meta = np.frombuffer(rec, dtype=np.uint8, count=512, offset=528).astype(np.int64).reshape(4, 128)
        base = meta & 0xF
        width = meta >> 4
        word_at = 1040
    words = np.frombuffer(rec, dtype="<u4", count=total_words, offset=word_at).astype(np.uint64)
    if raw:
        a = unpack_raw_fragment(words, bits)
        codes = a.T.copy() if is_v else a
        return ParsedRecord(raw, is_v, bits, mn, sc, base, width, codes, gws)
    codes = np.zeros((128, 128), np.int64)
    at = 0
    for g in range(4):
        if at != gws[g]:
            raise ValueError("group_word_start does not match the unit widths")
        for c in range(128):
            w = int(width[g, c])
            codes[32 * g:32 * g + 32, c] = base[g, c] + unpack_unit(words[at:at + w], w)
            at += w
    if at != total_words:
        raise ValueError("total_words does not match the unit widths")
    return ParsedRecord(raw, is_v, bits, mn, sc, base, width, codes, gws)


# ----------------------------------------------------------------------------
# Format variants, for the compression ablation only ([Fig. 2] step 2 and [Fig. 3]:
# the packing exploits quantized codes that concentrate on few values).  The
# library writes format v1 (frame-of-reference units, fp16 parameters, one meta
# byte per unit); these give the record size the alternatives would have.
# ----------------------------------------------------------------------------
VARIANT_V1 = "v1"                      # frame of reference (base = min), fp16 params, 8-bit meta
VARIANT_WIDTH_ONLY = "width-only"      # no base: w = bitlen(max code), meta holds w only
VARIANT_FP32_PARAMS = "fp32-params"    # min and scale stored as fp32 (1024 B instead of 512)
VARIANT_META4 = "meta4"                # b = 2: base and width in 2 bits each, 4-bit meta (256 B)


def record_bytes_variant(codes_slot: np.ndarray, bits: int, variant: str) -> int:
    """Bytes of one record of codes [slot, channel] under a format variant: the packed
    size, or the raw size of that variant when packing does not make it smaller."""
    codes_slot = np.asarray(codes_slot, dtype=np.int64)
    params = 1024 if variant == VARIANT_FP32_PARAMS else 512
    meta = 256 if variant == VARIANT_META4 else 512
    if variant == VARIANT_META4 and bits != 2:
        raise ValueError("the 4-bit meta variant is for 2-bit codes")
    wsum = 0
    for g in range(GROUPS_PER_BLOCK):
        for c in range(HEAD_DIM):
            unit = codes_slot[32 * g:32 * g + 32, c]
            if variant == VARIANT_WIDTH_ONLY:
                wsum += int(unit.max()).bit_length()
            else:
                wsum += unit_base_width(unit)[1]
    packed = _ceil16(16 + params + meta + 4 * wsum)
    raw = 16 + params + 2048 * bits
    return min(packed, raw)


# Records of the two layout variants (ablation only; the library writes and reads v1).
# The header is v1's with a variant id in flags bits 24-27; then
#   fp32 parameters: min[128] and scale[128] as fp32 (the fp16 values widened, so codes
#     and decoded values equal v1's), meta at 1040, words at 1552 (raw: words at 1040);
#   4-bit meta (b = 2): unit (g, c) in the 4-bit entry (byte (128 g + c) / 2, low
#     nibble for even c) = base | w << 2, meta at 528 (256 B), words at 784 (raw: as v1).
# Units, slices, the raw fragment order and the raw rule (packed >= raw size) are v1's.
VARIANT_IDS = {VARIANT_FP32_PARAMS: 1, VARIANT_META4: 2}


def build_record_variant(codes_slot: np.ndarray, mn16: np.ndarray, sc16: np.ndarray, bits: int,
                         is_v: bool, variant: str) -> bytes:
    """One record of a layout variant (v1 and width-only: build_record)."""
    if variant == VARIANT_V1:
        return build_record(codes_slot, mn16, sc16, bits, is_v)
    if variant == VARIANT_WIDTH_ONLY:
        return build_record(codes_slot, mn16, sc16, bits, is_v, UNITS_WIDTH_ONLY)
    if variant == VARIANT_META4 and bits != 2:
        raise ValueError("the 4-bit meta variant is for 2-bit codes")
    codes_slot = np.asarray(codes_slot, dtype=np.int64)
    fp32 = variant == VARIANT_FP32_PARAMS
    params = 1024 if fp32 else 512
    meta_bytes = 256 if variant == VARIANT_META4 else 512
    base = np.zeros((GROUPS_PER_BLOCK, HEAD_DIM), dtype=np.int64)
    width = np.zeros((GROUPS_PER_BLOCK, HEAD_DIM), dtype=np.int64)
    for g in range(GROUPS_PER_BLOCK):
        for c in range(HEAD_DIM):
            base[g, c], width[g, c] = unit_base_width(codes_slot[32 * g:32 * g + 32, c])
    raw_size = 16 + params + 2048 * bits
    raw = _ceil16(16 + params + meta_bytes + 4 * int(width.sum())) >= raw_size
    if raw:
        base[:] = 0
        width[:] = bits
        words = pack_raw_fragment(codes_slot.T if is_v else codes_slot, bits)
    else:
        words = np.concatenate([pack_unit(codes_slot[32 * g:32 * g + 32, c] - base[g, c], int(width[g, c]))
                                for g in range(GROUPS_PER_BLOCK) for c in range(HEAD_DIM)]).astype(np.uint32)
    group_start = [int(width[:g].sum()) for g in range(GROUPS_PER_BLOCK)]
    flags = ((RAW_FLAG if raw else 0) | (V_FLAG if is_v else 0) | (FORMAT_VERSION << 8) | (bits << 16)
             | (VARIANT_IDS[variant] << 24))
    out = bytearray()
    out += struct.pack("<4H", *group_start)
    out += struct.pack("<II", flags, int(words.size))
    pdt = np.float32 if fp32 else np.float16
    out += np.asarray(mn16, np.float16).astype(pdt).tobytes()
    out += np.asarray(sc16, np.float16).astype(pdt).tobytes()
    if not raw:
        if variant == VARIANT_META4:
            e = (base | (width << 2)).reshape(-1)
            out += (e[0::2] | (e[1::2] << 4)).astype(np.uint8).tobytes()
        else:
            out += (base | (width << 4)).astype(np.uint8).tobytes()
    out += words.astype("<u4").tobytes()
    out += b"\x00" * (_ceil16(len(out)) - len(out))
    assert raw == (len(out) == raw_size)
    return bytes(out)


def parse_record_variant(rec: bytes) -> ParsedRecord:
    """Inverse of build_record_variant for the two layout variants."""
    gws = list(struct.unpack_from("<4H", rec, 0))
    flags, total_words = struct.unpack_from("<II", rec, 8)
    vid = flags >> 24
    variant = {i: v for v, i in VARIANT_IDS.items()}.get(vid)
    if variant is None or (flags >> 8) & 0xFF != FORMAT_VERSION:
        raise ValueError("not a layout-variant record")
    raw, is_v, bits = bool(flags & RAW_FLAG), bool(flags & V_FLAG), (flags >> 16) & 0xF
    fp32 = variant == VARIANT_FP32_PARAMS
    pdt, params = ("<f4", 1024) if fp32 else ("<f2", 512)
    mn = np.frombuffer(rec, dtype=pdt, count=128, offset=16).astype(np.float16)
    sc = np.frombuffer(rec, dtype=pdt, count=128, offset=16 + params // 2).astype(np.float16)
    if raw:
        words = np.frombuffer(rec, dtype="<u4", count=total_words, offset=16 + params).astype(np.uint64)
        a = unpack_raw_fragment(words, bits)
        codes = a.T.copy() if is_v else a
        return ParsedRecord(raw, is_v, bits, mn, sc, np.zeros((4, 128), np.int64), np.full((4, 128), bits, np.int64),
                            codes, gws)
    if variant == VARIANT_META4:
        m = np.frombuffer(rec, dtype=np.uint8, count=256, offset=16 + params).astype(np.int64)
        e = np.stack([m & 0xF, m >> 4], axis=1).reshape(4, 128)
        base, width, word_at = e & 3, e >> 2, 16 + params + 256
    else:
        meta = np.frombuffer(rec, dtype=np.uint8, count=512, offset=16 + params).astype(np.int64).reshape(4, 128)
        base, width, word_at = meta & 0xF, meta >> 4, 16 + params + 512
    words = np.frombuffer(rec, dtype="<u4", count=total_words, offset=word_at).astype(np.uint64)
    codes = np.zeros((128, 128), np.int64)
    at = 0
    for g in range(4):
        if at != gws[g]:
            raise ValueError("group_word_start does not match the unit widths")
        for c in range(128):
            w = int(width[g, c])
            codes[32 * g:32 * g + 32, c] = base[g, c] + unpack_unit(words[at:at + w], w)
            at += w
    return ParsedRecord(raw, is_v, bits, mn, sc, base, width, codes, gws)


def block_codes(k_blk: np.ndarray, v_blk: np.ndarray, bits: int, key_kind: int = KEY_K_SUM):
    """Codes of one block in storage order (K [slot, channel], V [slot, channel])."""
    ck, _, _ = quantize_block_k(k_blk, bits)
    cv, _, _ = quantize_block_v(v_blk, bits)
    rank = stable_rank(reorder_keys(ck, cv, key_kind))
    perm = np.empty(BLOCK_TOKENS, dtype=np.int64)
    perm[rank] = np.arange(BLOCK_TOKENS)
    return ck[perm], cv[perm]


# ----------------------------------------------------------------------------
# One block: quantize -> reorder -> pack
# ----------------------------------------------------------------------------
def encode_block(k_blk: np.ndarray, v_blk: np.ndarray, bits: int, key_kind: int = KEY_K_SUM,
                 unit_mode: int = UNITS_FOR):
    """Encode one 128-token block of K and V.  Returns (k_record, v_record, perm)
    where perm[slot] = original token index within the block."""
    ck, k_mn, k_sc = quantize_block_k(k_blk, bits)
    cv, v_mn, v_sc = quantize_block_v(v_blk, bits)
    rank = stable_rank(reorder_keys(ck, cv, key_kind))
    perm = np.empty(BLOCK_TOKENS, dtype=np.int64)
    perm[rank] = np.arange(BLOCK_TOKENS)
    k_rec = build_record(ck[perm], k_mn, k_sc, bits, is_v=False, unit_mode=unit_mode)
    v_rec = build_record(cv[perm], v_mn[perm], v_sc[perm], bits, is_v=True, unit_mode=unit_mode)
    return k_rec, v_rec, perm


def dequant_k(rec: ParsedRecord) -> np.ndarray:
    """k_hat[slot, c] = mn_c + scale_c * code, fp64 (exact for fp16 params)."""
    return rec.mn.astype(np.float64)[None, :] + rec.scale.astype(np.float64)[None, :] * rec.codes


def dequant_v(rec: ParsedRecord) -> np.ndarray:
    """v_hat[slot, c] = mn_slot + scale_slot * code, fp64."""
    return rec.mn.astype(np.float64)[:, None] + rec.scale.astype(np.float64)[:, None] * rec.codes


# ----------------------------------------------------------------------------
# The cache: arenas, index, tail (packed-cache format v1, section 5)
# ----------------------------------------------------------------------------
class OracleCache:
    """Mirror of the packed cache state: two arenas, two index tables, the tail."""

    def __init__(self, batch, kv_heads, max_blocks, bits, key_kind=KEY_K_SUM, head_dim=HEAD_DIM,
                 unit_mode=UNITS_FOR):
        assert head_dim == HEAD_DIM
        self.batch, self.kv_heads, self.max_blocks = batch, kv_heads, max_blocks
        self.bits, self.key_kind, self.unit_mode = bits, key_kind, unit_mode
        self.k_arena = bytearray()
        self.v_arena = bytearray()
        self.k_index = np.zeros((batch, kv_heads, max_blocks, 2), np.uint32)
        self.v_index = np.zeros((batch, kv_heads, max_blocks, 2), np.uint32)
        self.perm = np.zeros((batch, kv_heads, max_blocks, BLOCK_TOKENS), np.uint8)
        self.n_blocks = 0
        self.tail_len = 0
        self.k_tail = np.zeros((batch, kv_heads, BLOCK_TOKENS, HEAD_DIM), np.float16)
        self.v_tail = np.zeros((batch, kv_heads, BLOCK_TOKENS, HEAD_DIM), np.float16)
        self._decoded = {}      # (tensor, b, h, block) -> fp64 [128, D]; records never change once written

    def encode_blocks(self, k: np.ndarray, v: np.ndarray, n_blocks: int, blocks=None):
        """Append n_blocks blocks per (batch, head); k, v: [B, Hkv, n_blocks*128, D] fp16.
        Records go to the arenas in ascending (b, h, block) order.  `blocks`
        optionally restricts which (b, h, i) triples are encoded (for sampled
        checks of large inputs; the arena layout is then not the full one)."""
        if self.n_blocks + n_blocks > self.max_blocks:
            raise ValueError("capacity")
        for b in range(self.batch):
            for h in range(self.kv_heads):
                for i in range(n_blocks):
                    if blocks is not None and (b, h, i) not in blocks:
                        continue
                    sl = slice(i * BLOCK_TOKENS, (i + 1) * BLOCK_TOKENS)
                    k_rec, v_rec, perm = encode_block(k[b, h, sl], v[b, h, sl], self.bits, self.key_kind,
                                                      self.unit_mode)
                    j = self.n_blocks + i
                    self.k_index[b, h, j] = (len(self.k_arena) // 16, len(k_rec) // 16)
                    self.v_index[b, h, j] = (len(self.v_arena) // 16, len(v_rec) // 16)
                    self.k_arena += k_rec
                    self.v_arena += v_rec
                    self.perm[b, h, j] = perm
        self.n_blocks += n_blocks

    def append_token(self, k_tok: np.ndarray, v_tok: np.ndarray):
        """k_tok, v_tok: [B, Hkv, D] fp16.  Encodes the tail when it reaches 128 tokens."""
        self.k_tail[:, :, self.tail_len] = k_tok
        self.v_tail[:, :, self.tail_len] = v_tok
        self.tail_len += 1
        if self.tail_len == BLOCK_TOKENS:
            self.encode_blocks(self.k_tail.copy(), self.v_tail.copy(), 1)
            self.tail_len = 0

    def record(self, which: str, b: int, h: int, i: int) -> bytes:
        arena, index = (self.k_arena, self.k_index) if which == "k" else (self.v_arena, self.v_index)
        off, ln = (int(x) for x in index[b, h, i])
        return bytes(arena[off * 16:(off + ln) * 16])

    def decoded(self, which: str, b: int, h: int) -> np.ndarray:
        """All tokens of (b, h) in storage order, decoded to fp64 [T, D]: blocks then tail."""
        parts = []
        for i in range(self.n_blocks):
            key = (which, b, h, i)
            if key not in self._decoded:
                rec = parse_record(self.record(which, b, h, i))
                self._decoded[key] = dequant_k(rec) if which == "k" else dequant_v(rec)
            parts.append(self._decoded[key])
        tail = (self.k_tail if which == "k" else self.v_tail)[b, h, :self.tail_len]
        parts.append(tail.astype(np.float64))
        return np.concatenate(parts, axis=0)

    @property
    def tokens(self) -> int:
        return self.n_blocks * BLOCK_TOKENS + self.tail_len


# ----------------------------------------------------------------------------
# Ragged batches and paged blocks (the visualisation page, "Read the caveat":
# paging and multi-request scheduling are what deployment adds)
# ----------------------------------------------------------------------------
class RaggedOracleCache(OracleCache):
    """A batch whose sequences have their own lengths, over the same record format.

    Sequence b holds seq_blocks[b] packed blocks and seq_tail[b] tail tokens.  Logical
    block j of sequence b lives at physical block p = table[b, j] (default
    b * max_blocks + j), i.e. at index entry (p // max_blocks, head, p % max_blocks):
    sequences may share a physical block (a common prefix) and a sequence's blocks need
    not be contiguous.  Calls append records to the arenas in ascending (sequence, head,
    block) order of the sequences they touch, as the uniform cache does.
    """

    def __init__(self, batch, kv_heads, max_blocks, bits, key_kind=KEY_K_SUM, table=None, unit_mode=UNITS_FOR):
        super().__init__(batch, kv_heads, max_blocks, bits, key_kind, unit_mode=unit_mode)
        self.seq_blocks = [0] * batch
        self.seq_tail = [0] * batch
        ids = np.arange(batch * max_blocks, dtype=np.int64).reshape(batch, max_blocks)
        self.table = ids if table is None else np.asarray(table, np.int64).reshape(batch, max_blocks)

    def physical(self, b: int, j: int):
        """(index row, block slot) of logical block j of sequence b."""
        return divmod(int(self.table[b, j]), self.max_blocks)

    def _encode_one(self, b, h, j, k_blk, v_blk):
        k_rec, v_rec, perm = encode_block(k_blk, v_blk, self.bits, self.key_kind, self.unit_mode)
        rb, jb = self.physical(b, j)
        self.k_index[rb, h, jb] = (len(self.k_arena) // 16, len(k_rec) // 16)
        self.v_index[rb, h, jb] = (len(self.v_arena) // 16, len(v_rec) // 16)
        self.k_arena += k_rec
        self.v_arena += v_rec
        self.perm[rb, h, jb] = perm
        for key in [key for key in self._decoded if key[1:] == (rb, h, jb)]:
            del self._decoded[key]

    def encode_blocks_ragged(self, k: np.ndarray, v: np.ndarray, n_blocks: int):
        """Append n_blocks blocks to every sequence (after its own blocks; its tail must
        be empty); k, v: [B, Hkv, n_blocks*128, D] fp16."""
        for b in range(self.batch):
            if self.seq_tail[b] != 0 or self.seq_blocks[b] + n_blocks > self.max_blocks:
                raise ValueError("tail not empty or capacity")
        for b in range(self.batch):
            for h in range(self.kv_heads):
                for i in range(n_blocks):
                    sl = slice(i * BLOCK_TOKENS, (i + 1) * BLOCK_TOKENS)
                    self._encode_one(b, h, self.seq_blocks[b] + i, k[b, h, sl], v[b, h, sl])
            self.seq_blocks[b] += n_blocks

    def append_token_ragged(self, k_tok: np.ndarray, v_tok: np.ndarray, active=None):
        """One token for every sequence in `active` (default: all), at its own tail
        position; a tail that reaches 128 tokens is encoded as the sequence's next block
        (sequences in ascending order)."""
        seqs = range(self.batch) if active is None else sorted(active)
        done = []
        for b in seqs:
            self.k_tail[b, :, self.seq_tail[b]] = k_tok[b]
            self.v_tail[b, :, self.seq_tail[b]] = v_tok[b]
            self.seq_tail[b] += 1
            if self.seq_tail[b] == BLOCK_TOKENS:
                done.append(b)
        for b in done:
            if self.seq_blocks[b] >= self.max_blocks:
                raise ValueError("capacity")
            for h in range(self.kv_heads):
                self._encode_one(b, h, self.seq_blocks[b], self.k_tail[b, h].copy(), self.v_tail[b, h].copy())
            self.seq_blocks[b] += 1
            self.seq_tail[b] = 0

    def seq_tokens(self, b: int) -> int:
        return self.seq_blocks[b] * BLOCK_TOKENS + self.seq_tail[b]

    def decoded(self, which: str, b: int, h: int) -> np.ndarray:
        """Sequence b, head h in storage order, fp64 [T_b, D]: its blocks through the
        table, then its tail."""
        parts = []
        for j in range(self.seq_blocks[b]):
            rb, jb = self.physical(b, j)
            key = (which, rb, h, jb)
            if key not in self._decoded:
                rec = parse_record(self.record(which, rb, h, jb))
                self._decoded[key] = dequant_k(rec) if which == "k" else dequant_v(rec)
            parts.append(self._decoded[key])
        tail = (self.k_tail if which == "k" else self.v_tail)[b, h, :self.seq_tail[b]]
        parts.append(tail.astype(np.float64))
        return np.concatenate(parts, axis=0)

    @property
    def tokens(self) -> int:
        return max(self.seq_tokens(b) for b in range(self.batch))


def ragged_qk(cache: RaggedOracleCache, q: np.ndarray, scale: float):
    """Scores of a ragged batch: [B, Hq, T_max] with row (b, hq) defined on [0, T_b)
    (NaN past it), and the sums of |terms|."""
    B, Hq, _ = q.shape
    G = Hq // cache.kv_heads
    T = cache.tokens
    scores = np.full((B, Hq, T), np.nan)
    sums = np.full((B, Hq, T), np.nan)
    for b in range(B):
        Tb = cache.seq_tokens(b)
        for h in range(cache.kv_heads):
            s_, a_ = qk_scores(q[b, h * G:(h + 1) * G], cache.decoded("k", b, h), scale)
            scores[b, h * G:(h + 1) * G, :Tb] = s_
            sums[b, h * G:(h + 1) * G, :Tb] = a_
    return scores, sums


def ragged_pv(cache: RaggedOracleCache, p: np.ndarray):
    """Outputs of a ragged batch: p [B, Hq, >= T_b] (only [:T_b] of row b is read)."""
    B, Hq, _ = p.shape
    G = Hq // cache.kv_heads
    out = np.zeros((B, Hq, HEAD_DIM))
    sums = np.zeros((B, Hq, HEAD_DIM))
    for b in range(B):
        Tb = cache.seq_tokens(b)
        for h in range(cache.kv_heads):
            o, a_ = pv_out(p[b, h * G:(h + 1) * G, :Tb], cache.decoded("v", b, h))
            out[b, h * G:(h + 1) * G] = o
            sums[b, h * G:(h + 1) * G] = a_
    return out, sums


def ragged_attention(cache: RaggedOracleCache, q: np.ndarray, scale: float):
    """Decode attention of a ragged batch: each sequence's softmax runs over its own
    T_b tokens ([Fig. 1])."""
    B, Hq, _ = q.shape
    scores, _ = ragged_qk(cache, q, scale)
    p = np.zeros_like(scores)
    for b in range(B):
        Tb = cache.seq_tokens(b)
        if Tb:  # a sequence with no tokens attends to nothing: its output is zero
            p[b, :, :Tb] = softmax(scores[b, :, :Tb])
    return ragged_pv(cache, p)


# ----------------------------------------------------------------------------
# The two decode products ([Fig. 1], [Fig. 2] fused decompression + GEMV), fp64
# ----------------------------------------------------------------------------
def qk_scores(q: np.ndarray, k_dec: np.ndarray, scale: float):
    """scores[i] = scale * sum_c q[c] * k_dec[i, c]; also sum_c |scale*q[c]*k_dec[i, c]|.
    q: [Hg, D] (the query heads of one kv head), k_dec: [T, D] fp64."""
    q64 = np.asarray(q, np.float64)
    k64 = np.asarray(k_dec, np.float64)
    terms = scale * q64[:, None, :] * k64[None, :, :]
    return terms.sum(axis=2), np.abs(terms).sum(axis=2)


def pv_out(p: np.ndarray, v_dec: np.ndarray):
    """out[c] = sum_i p[i] * v_dec[i, c]; also sum_i |p[i] * v_dec[i, c]|.
    p: [Hg, T], v_dec: [T, D] fp64."""
    p64 = np.asarray(p, np.float64)
    v64 = np.asarray(v_dec, np.float64)
    terms = p64[:, :, None] * v64[None, :, :]
    return terms.sum(axis=1), np.abs(terms).sum(axis=1)


def cache_qk(cache: OracleCache, q: np.ndarray, scale: float):
    """Scores for every (b, hq) of a cache: q [B, Hq, D] -> scores, abs_sums [B, Hq, T]."""
    B, Hq, _ = q.shape
    G = Hq // cache.kv_heads
    scores = np.zeros((B, Hq, cache.tokens))
    sums = np.zeros((B, Hq, cache.tokens))
    for b in range(B):
        for h in range(cache.kv_heads):
            kd = cache.decoded("k", b, h)
            s, a = qk_scores(q[b, h * G:(h + 1) * G], kd, scale)
            scores[b, h * G:(h + 1) * G] = s
            sums[b, h * G:(h + 1) * G] = a
    return scores, sums


def cache_pv(cache: OracleCache, p: np.ndarray):
    """Outputs for every (b, hq): p [B, Hq, T] (storage order) -> out, abs_sums [B, Hq, D]."""
    B, Hq, _ = p.shape
    G = Hq // cache.kv_heads
    out = np.zeros((B, Hq, HEAD_DIM))
    sums = np.zeros((B, Hq, HEAD_DIM))
    for b in range(B):
        for h in range(cache.kv_heads):
            vd = cache.decoded("v", b, h)
            o, a = pv_out(p[b, h * G:(h + 1) * G], vd)
            out[b, h * G:(h + 1) * G] = o
            sums[b, h * G:(h + 1) * G] = a
    return out, sums


def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    x = np.asarray(x, np.float64)
    m = x.max(axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=axis, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q k^T) v for one query vector, fp64 ([Fig. 1])."""
    s = scale * (np.asarray(k, np.float64) @ np.asarray(q, np.float64))
    return softmax(s) @ np.asarray(v, np.float64)


def cache_attention(cache: OracleCache, q: np.ndarray, scale: float):
    """Decode attention over the packed cache for every (b, hq): the scores, the
    softmax over all tokens of the sequence (packed blocks in storage order, then
    the tail) and the probability-weighted sum of the decoded values ([Fig. 1];
    [Fig. 2]: both products read the packed cache).  Returns out [B, Hq, D] and,
    per element, the sum of |p_i * v_hat_ic| (the scale of the parity tolerance).
    """
    scores, _ = cache_qk(cache, q, scale)
    return cache_pv(cache, softmax(scores))


def compression_ratio(n_tokens_total: int, arena_bytes: int, index_bytes: int) -> float:
    """fp16 bytes of one tensor / (record bytes + index bytes)."""
    return n_tokens_total * HEAD_DIM * 2 / float(arena_bytes + index_bytes)


def plain_quant_ratio(bits: int) -> float:
    """Same-b plain quantization baseline: codes + fp16 (min, scale) per row, no meta."""
    return BLOCK_TOKENS * HEAD_DIM * 2 / float(BLOCK_TOKENS * HEAD_DIM * bits / 8 + 512)

