"""Pins for the oracle's reorder, bit-packing and record layout (CPU only).

Format: packed-cache format v1, sections 2-4 (PackKV paper page, Figure 2 steps 1 and 2;
TL;DR: reorder with K and V bound together, light lossless encoding).
"""
import os
import re
import struct

import numpy as np
import pytest

import oracle as O
from decode_gemv_packkv_b200 import synth


def _lines(path):
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                yield line


def test_pack_unit_hand_words(golden_dir):
    for line in _lines(os.path.join(golden_dir, "pack_units.txt")):
        wtxt, rule, words = (t.strip() for t in line.split("|"))
        w = int(wtxt[2:])
        offs = np.array([eval(rule, {"j": j}) for j in range(32)], np.int64)  # rule text from the fixture
        want = [int(t, 16) for t in words.split()]
        got = O.pack_unit(offs, w)
        assert [int(x) for x in got] == want, line
        assert np.array_equal(O.unpack_unit(got, w), offs)


@pytest.mark.parametrize("w", [0, 1, 2, 3, 4])
def test_pack_round_trip_and_size(w):
    rng = np.random.default_rng(w)
    for _ in range(200):
        offs = rng.integers(0, 1 << w, 32) if w else np.zeros(32, np.int64)
        words = O.pack_unit(offs, w)
        assert words.shape == (w,)          # exactly w words: 32*w bits, no padding
        assert np.array_equal(O.unpack_unit(words, w), offs)


def test_unit_width_is_minimal():
    rng = np.random.default_rng(3)
    for _ in range(2000):
        codes = rng.integers(0, 16, 32) >> rng.integers(0, 5)
        codes = codes + rng.integers(0, 3)
        base, w = O.unit_base_width(codes)
        offs = codes - base
        assert base == codes.min()
        assert offs.max() < (1 << w)
        assert w == 0 or offs.max() >= (1 << (w - 1))


def test_stable_rank_matches_sorted():
    rng = np.random.default_rng(5)
    for trial in range(50):
        keys = rng.integers(0, 6 if trial % 2 else 10**6, 128)
        rank = O.stable_rank(keys)
        order = sorted(range(128), key=lambda t: keys[t])   # Python's sort is stable
        assert sorted(rank.tolist()) == list(range(128))
        assert [order[r] for r in range(128)] == list(np.argsort(rank))
        perm = np.empty(128, np.int64)
        perm[rank] = np.arange(128)
        assert np.all(np.diff(keys[perm]) >= 0)
        ties = np.diff(keys[perm]) == 0
        assert np.all(np.diff(perm)[ties] > 0)                  # ties keep index order
    assert np.array_equal(O.stable_rank(np.zeros(128, np.int64)), np.arange(128))


def _k1_block():
    k = np.full((128, 128), np.float16(0.5))
    k[:, 0] = (np.arange(128) % 2).astype(np.float16)
    return k


def _expand(txt):
    """Comma-separated hex items; `x*n` repeats an item, `[x,y]*n` a bracketed list."""
    vals = []
    for m in re.finditer(r"\[([^\]]*)\]\*(\d+)|([^,\[\]]+)", txt):
        if m.group(1) is not None:
            vals += [int(v, 16) for v in m.group(1).split(",")] * int(m.group(2))
        else:
            v, _, n = m.group(3).strip().partition("*")
            vals += [int(v, 16)] * (int(n) if n else 1)
    return vals


def _expected_record(spec):
    f = dict(t.strip().split("=", 1) for t in spec.split("|")[1:])
    out = bytearray()
    out += struct.pack("<4H", *[int(x) for x in f["gws"].split(",")])
    out += struct.pack("<II", int(f["flags"], 16), int(f["total_words"]))

    def expand16(txt):
        vals = _expand(txt)
        assert len(vals) == 128
        return struct.pack("<128H", *vals)
    out += expand16(f["min"]) + expand16(f["scale"])
    meta = bytearray(512)
    for item in f["meta"].split(","):
        where, val = item.split(":")
        g, c = where[1:].split("c")
        meta[int(g) * 128 + int(c)] = int(val, 16)
    out += meta
    if f["words"]:
        out += struct.pack(f"<{len(_expand(f['words']))}I", *_expand(f["words"]))
    out += b"\x00" * (int(f["len"]) - len(out))
    return bytes(out)


def test_records_hand_layout(golden_dir):
    specs = {line.split("|")[0].strip(): line for line in _lines(os.path.join(golden_dir, "records.txt"))}
    k = _k1_block()
    v = np.zeros((128, 128), np.float16)
    for key_kind, name in ((O.KEY_K_SUM, "K1_key1"), (O.KEY_IDENTITY, "K1_key0")):
        k_rec, _, perm = O.encode_block(k, v, 4, key_kind)
        assert k_rec == _expected_record(specs[name]), name
        if key_kind == O.KEY_K_SUM:
            assert perm.tolist() == list(range(0, 128, 2)) + list(range(1, 128, 2))
        else:
            assert perm.tolist() == list(range(128))


def _kv_block():
    """Block KV of the record goldens: K as block K1; V[t, c] = 1 for 1 <= c <= n_t with
    n_t = 2, 0, 1, 1 for t % 4 = 0, 1, 2, 3."""
    n = np.array([2, 0, 1, 1])[np.arange(128) % 4]
    v = (np.arange(128)[None, :] >= 1) & (np.arange(128)[None, :] <= n[:, None])
    return _k1_block(), v.astype(np.float16)


def test_records_kv_sum_key(golden_dir):
    """The K+V code-sum reorder key (key 2): permutation and both records by hand."""
    specs = {line.split("|")[0].strip(): line for line in _lines(os.path.join(golden_dir, "records.txt"))}
    k, v = _kv_block()
    k_rec, v_rec, perm = O.encode_block(k, v, 4, O.KEY_KV_SUM)
    want_perm = [int(x) for x in specs["KV_perm"].split("|")[1].split(",")]
    assert perm.tolist() == want_perm
    assert k_rec == _expected_record(specs["KV_key2_K"])
    assert v_rec == _expected_record(specs["KV_key2_V"])
    # the other keys order this block differently, so the golden pins the key itself
    assert O.encode_block(k, v, 4, O.KEY_K_SUM)[2].tolist() != want_perm
    assert O.encode_block(k, v, 4, O.KEY_IDENTITY)[2].tolist() != want_perm


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_raw_record_headers(golden_dir, bits):
    """Raw K and V records: header words (group_word_start, flags with the V bit,
    total_words) and length by hand; parse_record rejects a raw header that differs."""
    specs = {line.split("|")[0].strip(): line for line in _lines(os.path.join(golden_dir, "records.txt"))}
    k, v, _ = synth.small_case(70 + bits, 1, 1, 1, 128)
    k_rec, v_rec, _ = O.encode_block(k[0, 0], v[0, 0], bits)
    for rec, which in ((k_rec, "k"), (v_rec, "v")):
        f = dict(t.strip().split("=", 1) for t in specs[f"RAW_b{bits}_{which}"].split("|")[1:])
        assert len(rec) == int(f["len"])
        want = struct.pack("<4H", *[int(x) for x in f["gws"].split(",")]) + \
            struct.pack("<II", int(f["flags"], 16), int(f["total_words"]))
        assert rec[:16] == want, which
        for bad_at, bad in ((2, b"\x01\x00"), (12, b"\x00\x00\x00\x00")):
            broken = rec[:bad_at] + bad + rec[bad_at + len(bad):]
            with pytest.raises(ValueError):
                O.parse_record(broken)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("structured", [False, True])
def test_record_round_trip(bits, structured):
    k, v, _ = synth.small_case(40 + bits, 1, 1, 1, 256, structured=structured)
    for i in range(2):
        kb, vb = k[0, 0, 128 * i:128 * (i + 1)], v[0, 0, 128 * i:128 * (i + 1)]
        k_rec, v_rec, perm = O.encode_block(kb, vb, bits)
        ck, k_mn, k_sc = O.quantize_block_k(kb, bits)
        cv, v_mn, v_sc = O.quantize_block_v(vb, bits)
        pk, pv = O.parse_record(k_rec), O.parse_record(v_rec)
        assert np.array_equal(pk.codes, ck[perm]) and np.array_equal(pv.codes, cv[perm])
        assert np.array_equal(pk.mn.view(np.uint16), k_mn.view(np.uint16))
        assert np.array_equal(pv.scale.view(np.uint16), v_sc[perm].view(np.uint16))
        for rec, p in ((k_rec, pk), (v_rec, pv)):
            assert len(rec) % 16 == 0
            assert len(rec) <= O.record_bytes_max(bits)
            assert p.raw == (len(rec) == O.raw_record_bytes(bits))
            if not p.raw:
                assert len(rec) == -(-(1040 + 4 * int(p.width.sum())) // 16) * 16
                assert len(rec) < O.raw_record_bytes(bits)
            assert p.is_v == (rec is v_rec)
        # K-sum key: keys are non-decreasing in storage order
        keys = ck.astype(np.int64).sum(axis=1)
        assert np.all(np.diff(keys[perm]) >= 0)


def test_random_blocks_fall_back_to_raw():
    k, v, _ = synth.small_case(9, 1, 1, 1, 128)
    for bits in (2, 3, 4):
        k_rec, v_rec, _ = O.encode_block(k[0, 0], v[0, 0], bits)
        assert len(k_rec) == O.raw_record_bytes(bits) == len(v_rec)


def test_cache_append_equals_block_encode():
    """Growing the cache token by token yields the records of a block encode ([Abs]: growth)."""
    k, v, _ = synth.small_case(12, 2, 2, 1, 300)
    a = O.OracleCache(2, 2, 4, 3)
    a.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, 300):
        a.append_token(k[:, :, t], v[:, :, t])
    b = O.OracleCache(2, 2, 4, 3)
    for t in range(300):
        b.append_token(k[:, :, t], v[:, :, t])
    assert a.n_blocks == b.n_blocks == 2 and a.tail_len == b.tail_len == 44
    for bb in range(2):
        for h in range(2):
            for i in range(2):
                assert a.record("k", bb, h, i) == b.record("k", bb, h, i)
                assert a.record("v", bb, h, i) == b.record("v", bb, h, i)
    assert np.array_equal(a.k_tail[:, :, :44], b.k_tail[:, :, :44])
    # arena layout: ascending (b, h, block) within one encode call, offsets contiguous
    offs = a.k_index[:, :, :2, 0].reshape(-1)
    lens = a.k_index[:, :, :2, 1].reshape(-1)
    assert np.array_equal(a.k_index[:, :, :2, 0].transpose(0, 1, 2).reshape(-1),
                          np.concatenate([[0], np.cumsum(lens)[:-1]]))
    assert offs[-1] + lens[-1] == len(a.k_arena) // 16


def test_raw_fragment_order_hand_words(golden_dir):
    matrices = {"m+2k": lambda m, k: m + 2 * k, "m/8+k": lambda m, k: m // 8 + k}
    for line in _lines(os.path.join(golden_dir, "raw_fragment_words.txt")):
        bits, name, idx, want = (t.strip() for t in line.split("|"))
        bits, idx = int(bits), int(idx)
        a = np.fromfunction(lambda m, k: matrices[name](m, k) % (1 << bits), (128, 128), dtype=np.int64)
        assert int(O.pack_raw_fragment(a, bits)[idx]) == int(want, 16), line


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_raw_fragment_order_is_a_bijection(bits):
    """Every bit of every code has its own place and the word area is filled exactly."""
    seen = set()
    for m in range(128):
        for k in range(128):
            for w, bit, width, _ in O.frag_fields(bits, m, k):
                assert 0 <= w < 512 * bits and bit + width <= 32
                for i in range(width):
                    seen.add((w, bit + i))
    assert len(seen) == 128 * 128 * bits
    rng = np.random.default_rng(bits)
    a = rng.integers(0, 1 << bits, (128, 128))
    assert np.array_equal(O.unpack_raw_fragment(O.pack_raw_fragment(a, bits), bits), a)


def test_raw_v_record_stores_the_transpose():
    """In a V record the fragment rows are channels: word 0's first field is code[slot 0][channel 0],
    its rh field (row 8) is code[slot 0][channel 8], and byte 1 starts with code[slot 1][channel 0]."""
    k, v, _ = synth.small_case(31, 1, 1, 1, 128)
    _, v_rec, perm = O.encode_block(k[0, 0], v[0, 0], 4)
    assert len(v_rec) == O.raw_record_bytes(4)
    codes = O.quantize_block_v(v[0, 0], 4)[0][perm]      # [slot, channel]
    w0 = int(np.frombuffer(v_rec, "<u4", 1, 528)[0])
    assert w0 & 0xF == codes[0, 0] and (w0 >> 4) & 0xF == codes[0, 8] and (w0 >> 8) & 0xF == codes[1, 0]


def test_plain_quant_ratio_closed_form():
    """Plain b-bit quantization of a 128x128 fp16 block: 2*16384 bytes over the codes
    (16384*b/8) plus fp16 min and scale for 128 rows (512 bytes)."""
    assert O.plain_quant_ratio(4) == pytest.approx(32768 / 8704, rel=1e-15)
    assert O.plain_quant_ratio(3) == pytest.approx(32768 / 6656, rel=1e-15)
    assert O.plain_quant_ratio(2) == pytest.approx(32768 / 4608, rel=1e-15)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_compression_ratio_of_raw_and_packed_caches(bits):
    """i.i.d. Gaussian blocks never pack below b bits, so every record is raw and the
    ratio is exactly 32768 / (528 + 2048 b + 8) per block; run-structured blocks pack,
    their arena is smaller than all-raw, and with the identity key (runs kept in token
    order) the ratio beats plain quantization."""
    nb, T = 4, 4 * 128
    k, v, _ = synth.small_case(90 + bits, 1, 1, 1, T)
    oc = O.OracleCache(1, 1, nb, bits, O.KEY_K_SUM)
    oc.encode_blocks(k, v, nb)
    raw = O.raw_record_bytes(bits)
    assert len(oc.k_arena) == nb * raw and len(oc.v_arena) == nb * raw
    assert O.compression_ratio(T, len(oc.k_arena), nb * 8) == pytest.approx(32768 / (raw + 8), rel=1e-15)
    ks, vs, _ = synth.small_case(90 + bits, 1, 1, 1, T, structured=True)
    os_ = O.OracleCache(1, 1, nb, bits, O.KEY_IDENTITY)
    os_.encode_blocks(ks, vs, nb)
    for arena in (os_.k_arena, os_.v_arena):
        assert len(arena) < nb * raw
        assert O.compression_ratio(T, len(arena), nb * 8) > O.plain_quant_ratio(bits)
