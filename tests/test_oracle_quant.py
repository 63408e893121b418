"""Pins for the oracle's fp16 round-up and quantizer (CPU only).

Format: packed-cache format v1, section 1 (PackKV paper page, Figure 5 granularities;
Figure 2 / TL;DR quantization step).
"""
import bisect
import os

import numpy as np
import pytest

import oracle as O


def _parse_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line)
    return rows


def _all_nonneg_fp16():
    bits = np.arange(0, 0x7C00, dtype=np.uint16)           # +0 .. 65504
    vals = bits.view(np.float16).astype(np.float64)
    return bits, vals


def test_fp16_round_up_hand_table(golden_dir):
    for line in _parse_golden(os.path.join(golden_dir, "fp16_round_up.txt")):
        xin, want = (int(t, 16) for t in line.split())
        x = np.array([xin], np.uint32).view(np.float32)
        got = O.fp16_round_up(x).view(np.uint16)[0]
        assert got == want, (hex(xin), hex(got), hex(want))


def test_fp16_round_up_brute_force():
    """Smallest binary16 >= x by binary search over the sorted list of all
    nonnegative finite binary16 values (an enumeration, not the formula)."""
    bits, vals = _all_nonneg_fp16()
    rng = np.random.default_rng(7)
    xs = [rng.uniform(0, 70000, 4000), np.exp2(rng.uniform(-30, 16, 4000))]
    # every binary16 value and its fp32 neighbours
    v32 = vals.astype(np.float32)
    xs += [v32, np.nextafter(v32, np.float32(np.inf)), np.nextafter(v32, np.float32(0))]
    x = np.concatenate([np.asarray(a, np.float32) for a in xs])
    x = x[np.isfinite(x) & (x >= 0)]
    got = O.fp16_round_up(x)
    vl = list(vals)
    for xi, gi in zip(x.astype(np.float64), got.astype(np.float64)):
        k = bisect.bisect_left(vl, xi)
        want = vl[k] if k < len(vl) else np.inf
        assert gi == want, (xi, gi, want)


def test_quant_rows_hand_examples(golden_dir):
    for line in _parse_golden(os.path.join(golden_dir, "quant_rows.txt")):
        name, bits, pad, values, mn, sc, codes = (t.strip() for t in line.split("|"))
        bits = int(bits)
        vals = [float(v) for v in values.split(",")]
        row = np.full(128, np.float16(float(pad)), np.float16)
        row[:len(vals)] = np.array(vals, np.float16)
        c, m, s = O.quantize_rows(row[None, :], bits)
        listed, pad_code = codes.split(";")
        want = [int(t) for t in listed.split(",")]
        assert list(c[0, :len(want)]) == want, name
        assert np.all(c[0, len(vals):] == int(pad_code)), name
        assert m.view(np.uint16)[0] == int(mn, 16), name
        assert s.view(np.uint16)[0] == int(sc, 16), name


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quant_error_bound_and_extremes(bits):
    rng = np.random.default_rng(bits)
    x = (rng.standard_normal((300, 128)) * np.exp2(rng.uniform(-12, 10, (300, 1)))
         + rng.standard_normal((300, 1)) * 3).astype(np.float16)
    codes, mn, sc = O.quantize_rows(x, bits)
    qmax = (1 << bits) - 1
    assert codes.max() <= qmax
    xh = mn.astype(np.float64)[:, None] + sc.astype(np.float64)[:, None] * codes
    err = np.abs(xh - x.astype(np.float64))
    assert np.all(err <= O.quant_error_bound(sc, bits)[:, None])
    # the minimum is coded exactly as 0; the maximum as 2^b-1 when the scale is normal
    assert np.all(codes[np.arange(300), x.argmin(axis=1)] == 0)
    normal = sc.astype(np.float64) >= 2.0 ** -14
    assert np.all(codes[np.arange(300), x.argmax(axis=1)][normal] == qmax)
    # scale is the smallest binary16 >= s, so s <= scale < s * (1 + 2^-10) for normal scales
    s = (x.max(axis=1).astype(np.float32) - mn.astype(np.float32)) / np.float32(qmax)
    assert np.all(sc.astype(np.float64) >= s.astype(np.float64))
    assert np.all(sc.astype(np.float64)[normal] <= s.astype(np.float64)[normal] * (1 + 2.0 ** -10))


def test_quant_subnormal_scales():
    """Tiny ranges give subnormal fp16 scales; the bound still holds and codes stay in range."""
    rng = np.random.default_rng(11)
    ticks = rng.integers(0, 40, (200, 128))
    x = (ticks * 2.0 ** -24).astype(np.float16)
    for bits in (2, 3, 4):
        codes, mn, sc = O.quantize_rows(x, bits)
        assert codes.max() <= (1 << bits) - 1
        xh = mn.astype(np.float64)[:, None] + sc.astype(np.float64)[:, None] * codes
        assert np.all(np.abs(xh - x.astype(np.float64)) <= O.quant_error_bound(sc, bits)[:, None])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quant_grid_inputs_decode_exactly(bits):
    """x = m + 2^e * n with integer n spanning {0, .., 2^b-1}: the quantizer recovers n."""
    rng = np.random.default_rng(20 + bits)
    qmax = (1 << bits) - 1
    n = rng.integers(0, qmax + 1, (64, 128))
    n[:, 0], n[:, 1] = 0, qmax
    e = rng.integers(-6, 3, (64, 1)).astype(np.float64)
    m = rng.integers(-100, 100, (64, 1)) * np.exp2(e)      # m on the same 2^e grid
    x = (m + np.exp2(e) * n).astype(np.float16)
    assert np.array_equal(x.astype(np.float64), m + np.exp2(e) * n)  # on the fp16 grid
    codes, mn, sc = O.quantize_rows(x, bits)
    assert np.array_equal(codes, n)
    assert np.array_equal(sc.astype(np.float64), np.exp2(e)[:, 0])


def test_quant_constant_rows_and_granularity():
    k = np.full((128, 128), np.float16(1.25))
    k[:, 3] = np.arange(128, dtype=np.float16) / np.float16(64)     # one varying channel
    codes, mn, sc = O.quantize_block_k(k, 4)
    assert codes.shape == (128, 128)
    assert np.all(sc[np.arange(128) != 3] == 0) and sc[3] > 0
    assert np.all(codes[:, np.arange(128) != 3] == 0)
    # V is per token: the same block quantized token-wise has one live row per token
    codes_v, mn_v, sc_v = O.quantize_block_v(k, 4)
    assert np.all(sc_v > 0) or np.all(mn_v <= np.float16(1.25))
    assert codes_v.shape == (128, 128)
    assert np.array_equal(codes_v, O.quantize_rows(k, 4)[0])
    assert np.array_equal(codes, O.quantize_rows(k.T, 4)[0].T)
