"""Format variants for the compression ablation (CPU only): width-only units, fp32
parameters and 4-bit meta for 2-bit codes, against the library's format v1.

PackKV paper page, Figure 2 step (2) (bit-packing after the reorder) and Figure 3
(the quantized integers concentrate on few values, which is what frame-of-
reference units and narrow meta exploit).  The oracle's size model of each
variant is pinned to the real v1 records and to record sizes derived by hand;
the ratios it gives on the synthetic workloads are reported by the last test.
"""
import struct

import numpy as np
import pytest

import oracle as O
from decode_gemv_packkv_b200 import synth


def test_v1_size_model_matches_the_records():
    for bits in (2, 3, 4):
        for structured in (False, True):
            k, v, _ = synth.small_case(70 + bits, 1, 1, 1, 256, structured=structured)
            for i in range(2):
                kb, vb = k[0, 0, 128 * i:128 * (i + 1)], v[0, 0, 128 * i:128 * (i + 1)]
                k_rec, v_rec, _ = O.encode_block(kb, vb, bits)
                ck, cv = O.block_codes(kb, vb, bits)
                assert O.record_bytes_variant(ck, bits, O.VARIANT_V1) == len(k_rec)
                assert O.record_bytes_variant(cv, bits, O.VARIANT_V1) == len(v_rec)


def test_variant_sizes_by_hand():
    """Block K1 of the record goldens (0.5 everywhere, channel 0 = t % 2), K-sum key:
    4-bit: every unit constant (units g2, g3 of channel 0 hold code 15) -> v1 1040 B;
    width-only needs 4 bits in those two units -> 1040 + 4*8 = 1072 B; fp32 params
    1040 + 512 = 1552 B.  2-bit: codes 0 / 3 -> v1 1040 B, width-only 2 bits in two
    units -> 1056 B, 4-bit meta 16 + 512 + 256 = 784 B."""
    k = np.full((128, 128), np.float16(0.5))
    k[:, 0] = (np.arange(128) % 2).astype(np.float16)
    v = np.zeros((128, 128), np.float16)
    ck4, _ = O.block_codes(k, v, 4)
    assert O.record_bytes_variant(ck4, 4, O.VARIANT_V1) == 1040
    assert O.record_bytes_variant(ck4, 4, O.VARIANT_WIDTH_ONLY) == 1072
    assert O.record_bytes_variant(ck4, 4, O.VARIANT_FP32_PARAMS) == 1552
    ck2, _ = O.block_codes(k, v, 2)
    assert O.record_bytes_variant(ck2, 2, O.VARIANT_V1) == 1040
    assert O.record_bytes_variant(ck2, 2, O.VARIANT_WIDTH_ONLY) == 1056
    assert O.record_bytes_variant(ck2, 2, O.VARIANT_META4) == 784
    with pytest.raises(ValueError):
        O.record_bytes_variant(ck4, 4, O.VARIANT_META4)


def test_width_only_records():
    """The encoder's width-only unit mode writes format v1 records (base 0, the width
    of the largest code): their lengths are the size model's, they decode to the
    same codes as the frame-of-reference records, and on block K1 of the record
    goldens (0.5 everywhere, channel 0 = t % 2, K-sum key, 4-bit) the two units of
    channel 0 in groups 2 and 3 carry meta byte 0x40 and four words 0xFFFFFFFF
    (frame of reference: meta 0x0F and no words)."""
    for bits in (2, 3, 4):
        for structured in (False, True):
            k, v, _ = synth.small_case(90 + bits, 1, 1, 1, 256, structured=structured)
            for i in range(2):
                kb, vb = k[0, 0, 128 * i:128 * (i + 1)], v[0, 0, 128 * i:128 * (i + 1)]
                kw, vw, pw = O.encode_block(kb, vb, bits, unit_mode=O.UNITS_WIDTH_ONLY)
                kf, vf, pf = O.encode_block(kb, vb, bits)
                assert np.array_equal(pw, pf)
                ck, cv = O.block_codes(kb, vb, bits)
                assert len(kw) == O.record_bytes_variant(ck, bits, O.VARIANT_WIDTH_ONLY)
                assert len(vw) == O.record_bytes_variant(cv, bits, O.VARIANT_WIDTH_ONLY)
                for a, b in ((kw, kf), (vw, vf)):
                    ra, rb = O.parse_record(a), O.parse_record(b)
                    assert np.array_equal(ra.codes, rb.codes)
                    if not ra.raw:
                        assert np.all(ra.base == 0)
    k = np.full((128, 128), np.float16(0.5))
    k[:, 0] = (np.arange(128) % 2).astype(np.float16)
    v = np.zeros((128, 128), np.float16)
    kw, _, _ = O.encode_block(k, v, 4, unit_mode=O.UNITS_WIDTH_ONLY)
    kf, _, _ = O.encode_block(k, v, 4)
    assert len(kw) == 1072 and len(kf) == 1040
    meta_w, meta_f = kw[528:1040], kf[528:1040]
    for g in range(4):
        assert meta_w[g * 128] == (0x40 if g >= 2 else 0x00)
        assert meta_f[g * 128] == (0x0F if g >= 2 else 0x00)
        assert all(meta_w[g * 128 + c] == 0 for c in range(1, 128))
    words = np.frombuffer(kw, "<u4", 8, 1040)
    assert np.all(words == 0xFFFFFFFF)


def test_layout_variant_records():
    """Records of the fp32-parameter and 4-bit-meta layouts: their lengths are the size
    model's, they parse back to the v1 codes and parameters, and v1's parser refuses
    them.  By hand, on block K1 of the record goldens (0.5 everywhere, channel 0 =
    t % 2, K-sum key): at 2 bits the units of channel 0 in groups 2 and 3 hold code 3,
    so their 4-bit entries (low nibble of meta bytes 128 and 192) are base 3 | w 0 << 2
    = 0x3 and the record is 784 bytes; at 4 bits the fp32 record is 1552 bytes with
    min[1] = 0.5f (0x3F000000) and meta byte 0x0F for those units."""
    for bits in (2, 3, 4):
        for structured in (False, True):
            k, v, _ = synth.small_case(110 + bits, 1, 1, 1, 128, structured=structured)
            kb, vb = k[0, 0], v[0, 0]
            ck, k_mn, k_sc = O.quantize_block_k(kb, bits)
            cv, v_mn, v_sc = O.quantize_block_v(vb, bits)
            rank = O.stable_rank(O.reorder_keys(ck, cv, O.KEY_K_SUM))
            perm = np.empty(128, np.int64)
            perm[rank] = np.arange(128)
            variants = [O.VARIANT_FP32_PARAMS] + ([O.VARIANT_META4] if bits == 2 else [])
            for codes, mn, sc, is_v in ((ck[perm], k_mn, k_sc, False), (cv[perm], v_mn[perm], v_sc[perm], True)):
                v1 = O.parse_record(O.build_record(codes, mn, sc, bits, is_v))
                for var in variants:
                    rec = O.build_record_variant(codes, mn, sc, bits, is_v, var)
                    assert len(rec) == O.record_bytes_variant(codes, bits, var)
                    p = O.parse_record_variant(rec)
                    assert np.array_equal(p.codes, codes) and np.array_equal(p.codes, v1.codes)
                    assert np.array_equal(p.mn, v1.mn) and np.array_equal(p.scale, v1.scale)
                    assert p.raw == v1.raw and p.is_v == is_v
                    with pytest.raises(ValueError):
                        O.parse_record(rec)
    k = np.full((128, 128), np.float16(0.5))
    k[:, 0] = (np.arange(128) % 2).astype(np.float16)
    ck, mn, sc = O.quantize_block_k(k, 2)
    rank = O.stable_rank(O.reorder_keys(ck, ck, O.KEY_K_SUM))
    perm = np.empty(128, np.int64)
    perm[rank] = np.arange(128)
    rec = O.build_record_variant(ck[perm], mn, sc, 2, False, O.VARIANT_META4)
    assert len(rec) == 784
    meta = rec[528:784]
    assert meta[128] == 0x03 and meta[192] == 0x03 and meta[0] == 0 and meta[64] == 0
    assert all(b == 0 for i, b in enumerate(meta) if i not in (128, 192))
    ck4, mn4, sc4 = O.quantize_block_k(k, 4)
    rank = O.stable_rank(O.reorder_keys(ck4, ck4, O.KEY_K_SUM))
    perm[rank] = np.arange(128)
    rec = O.build_record_variant(ck4[perm], mn4, sc4, 4, False, O.VARIANT_FP32_PARAMS)
    assert len(rec) == 1552
    assert struct.unpack_from("<I", rec, 16 + 4)[0] == 0x3F000000
    assert rec[1040 + 256] == 0x0F and rec[1040 + 384] == 0x0F


def test_variant_invariants():
    """Width-only units are never narrower than frame-of-reference ones; fp32 params
    add exactly 512 B to a packed record and to the raw size; 4-bit meta saves 256 B
    on a packed 2-bit record."""
    rng = np.random.default_rng(3)
    for trial in range(40):
        bits = int(rng.integers(2, 5))
        codes = rng.integers(0, 1 << bits, (128, 128)) >> rng.integers(0, bits + 1, (1, 128))
        codes = np.minimum(codes + rng.integers(0, 2, (1, 128)), (1 << bits) - 1)
        v1 = O.record_bytes_variant(codes, bits, O.VARIANT_V1)
        assert O.record_bytes_variant(codes, bits, O.VARIANT_WIDTH_ONLY) >= v1
        raw = 528 + 2048 * bits
        f32 = O.record_bytes_variant(codes, bits, O.VARIANT_FP32_PARAMS)
        if v1 < raw:
            assert f32 == v1 + 512
        else:
            assert f32 == raw + 512
        if bits == 2 and v1 < raw:  # both sizes round up to 16 B from values 256 B apart
            assert O.record_bytes_variant(codes, bits, O.VARIANT_META4) == v1 - 256


def _ratio(kind, bits, variant, key=O.KEY_K_SUM, n_blocks=8, seqs=2):
    tot_k = tot_v = 0
    for s in range(seqs):
        ks, vs = synth.kv_slice(1001, 32, 0, s, n_blocks * 128, structured=(kind == "structured"))
        for i in range(n_blocks):
            ck, cv = O.block_codes(ks[128 * i:128 * (i + 1)], vs[128 * i:128 * (i + 1)], bits, key)
            tot_k += O.record_bytes_variant(ck, bits, variant) + 8
            tot_v += O.record_bytes_variant(cv, bits, variant) + 8
    fp16 = seqs * n_blocks * 128 * 128 * 2
    return fp16 / tot_k, fp16 / tot_v


def test_variant_compression_report(capsys):
    """Compression ratios (fp16 bytes / (record + 8-B index entry)) of each variant on
    the synthetic inputs; the ordering the size model implies must hold."""
    rows = []
    for kind in ("i.i.d.", "structured"):
        for bits in (4, 2):
            base = _ratio(kind, bits, O.VARIANT_V1)
            rows.append((kind, bits, O.VARIANT_V1, *base))
            for var in (O.VARIANT_WIDTH_ONLY, O.VARIANT_FP32_PARAMS) + ((O.VARIANT_META4,) if bits == 2 else ()):
                r = _ratio(kind, bits, var)
                rows.append((kind, bits, var, *r))
                if var == O.VARIANT_META4:
                    assert r[0] >= base[0] and r[1] >= base[1]
                else:
                    assert r[0] <= base[0] + 1e-12 and r[1] <= base[1] + 1e-12
    with capsys.disabled():
        print("\ninputs | bits | variant | CR K | CR V")
        for row in rows:
            print("%s | %d | %s | %.3f | %.3f" % row)
