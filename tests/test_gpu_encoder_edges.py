"""GPU encoder on the quantizer's edge cases, bit-exact against the CPU oracle.

Random fp16 inputs almost never hit a rounding tie, a subnormal scale or an
fp16 scale that rounds up at a binade edge, so these blocks are built to hit
them (PackKV paper page, Figure 5 granularities and Figure 2 quantize step;
packed-cache format v1, section 1):
  * the hand-derived rows of tests/golden/quant_rows.txt (half-even ties, a
    scale rounded up, signed zeros, constant rows) placed in K channels (K is
    quantized per channel) and in V tokens (V is quantized per token);
  * rows whose values sit exactly half-way between two codes;
  * tiny ranges whose scale is an fp16 subnormal;
  * exactly gridded rows (x = m + 2^e * n), constant rows, rows of signed
    zeros and rows spanning the whole fp16 range.
Records, index, arena ends and permutations must match bit for bit, for every
code width and reorder key.
"""
import os

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import compare_encoder, to_dev

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "quant_rows.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            _, _, pad, values, *_ = (t.strip() for t in line.split("|"))
            row = np.full(128, np.float16(float(pad)), np.float16)
            vals = [float(v) for v in values.split(",")]
            row[:len(vals)] = np.array(vals, np.float16)
            rows.append(row)
    return rows


def _edge_rows(bits: int, rng: np.random.Generator):
    """128-value rows, each built to hit one edge of the quantizer at this code width."""
    qmax = (1 << bits) - 1
    rows = list(_golden_rows())
    # ties: min 0, max qmax (scale exactly 1), the rest at k + 1/2 (round half to even)
    for _ in range(4):
        r = (rng.integers(0, qmax, 128) + 0.5).astype(np.float16)
        r[0], r[1] = 0, qmax
        rows.append(r)
    # ties at a scale of 2^e: values on the half-grid of a power-of-two scale
    for e in (-9, -3, 4):
        r = ((rng.integers(0, 2 * qmax + 1, 128)) * 2.0 ** (e - 1)).astype(np.float16)
        r[0], r[1] = 0, qmax * 2.0 ** e
        rows.append(r)
    # tiny ranges: subnormal fp16 scales
    for top in (1, 3, 7, 40, 1023):
        rows.append((rng.integers(0, top + 1, 128) * 2.0 ** -24).astype(np.float16))
    # exactly gridded rows: m + 2^e * n decodes exactly
    for e in (-6, 0, 2):
        n = rng.integers(0, qmax + 1, 128)
        n[0], n[1] = 0, qmax
        m = rng.integers(-100, 100) * 2.0 ** e
        rows.append((m + 2.0 ** e * n).astype(np.float16))
    # constant rows, signed zeros, the whole fp16 range
    rows.append(np.full(128, np.float16(-3.5)))
    rows.append(np.where(rng.random(128) < 0.5, np.float16(-0.0), np.float16(0.0)).astype(np.float16))
    z = np.zeros(128, np.float16)
    z[5] = np.float16(-0.0)
    z[6] = np.float16(2.0 ** -24)
    rows.append(z)
    r = rng.standard_normal(128).astype(np.float16)
    r[3], r[4] = np.float16(-65504.0), np.float16(65504.0)
    rows.append(r)
    # scale rounding up at a binade edge: range / qmax just above a power of two
    for e in (-12, -2, 5):
        r = rng.uniform(0, 1, 128).astype(np.float16) * np.float16(2.0 ** e * qmax)
        r[0] = 0
        r[1] = np.float16(2.0 ** e * qmax) + np.float16(2.0 ** (e - 9))
        rows.append(r.astype(np.float16))
    return rows


def _edge_blocks(bits: int, n_blocks: int, seed: int):
    """K, V [n_blocks*128, 128]: the edge rows as K channels and as V tokens, the
    remaining channels / tokens ordinary Gaussian values."""
    rng = np.random.default_rng(seed)
    rows = _edge_rows(bits, rng)
    T = n_blocks * 128
    k = rng.standard_normal((T, 128)).astype(np.float16)
    v = rng.standard_normal((T, 128)).astype(np.float16)
    for i, r in enumerate(rows):
        blk, c = divmod(i, 96)        # up to 96 edge channels / tokens per block
        if blk >= n_blocks:
            break
        perm = rng.permutation(128)   # the edge values in a shuffled token / channel order
        k[blk * 128:(blk + 1) * 128, (c * 37) % 128] = r[perm]
        v[blk * 128 + (c * 53) % 128] = r[rng.permutation(128)]
    return k, v


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("key", [O.KEY_IDENTITY, O.KEY_K_SUM, O.KEY_KV_SUM])
def test_encoder_edge_rows_bit_exact(pk, bits, key):
    B, H, nb = 1, 2, 2
    k = np.empty((B, H, nb * 128, 128), np.float16)
    v = np.empty_like(k)
    for h in range(H):
        k[0, h], v[0, h] = _edge_blocks(bits, nb, 1000 * bits + 10 * key + h)
    assert np.all(np.isfinite(k)) and np.all(np.isfinite(v))
    cache = pk.PackKVCache(B, H, nb, bits, reorder_key=key, keep_perm=True)
    pk.packkv_encode_block(cache, to_dev(k), to_dev(v), nb)
    oc = O.OracleCache(B, H, nb, bits, key)
    oc.encode_blocks(k, v, nb)
    compare_encoder(cache, oc)
    assert pk.packkv_get_status(cache) == 0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_encoder_whole_blocks_of_one_edge(pk, bits):
    """Blocks made entirely of one kind of edge: all ties, all subnormal, all constant,
    all signed zeros, all on a grid (most units constant or narrow: compressed records)."""
    rng = np.random.default_rng(bits)
    qmax = (1 << bits) - 1
    blocks = []
    t = (rng.integers(0, qmax, (128, 128)) + 0.5).astype(np.float16)
    t[0], t[1] = 0, qmax
    blocks.append((t, t.T.copy()))
    sub = (rng.integers(0, 9, (128, 128)) * 2.0 ** -24).astype(np.float16)
    blocks.append((sub, sub[::-1].copy()))
    blocks.append((np.full((128, 128), np.float16(7.25)), np.full((128, 128), np.float16(-0.5))))
    zeros = np.where(rng.random((128, 128)) < 0.5, np.float16(-0.0), np.float16(0.0)).astype(np.float16)
    blocks.append((zeros, zeros.T.copy()))
    n = rng.integers(0, qmax + 1, (128, 128))
    grid = (np.float16(3.0) + np.float16(0.25) * n).astype(np.float16)
    blocks.append((grid, grid[:, ::-1].copy()))
    nb = len(blocks)
    k = np.concatenate([b[0] for b in blocks])[None, None]
    v = np.concatenate([b[1] for b in blocks])[None, None]
    for key in (O.KEY_IDENTITY, O.KEY_K_SUM, O.KEY_KV_SUM):
        cache = pk.PackKVCache(1, 1, nb, bits, reorder_key=key, keep_perm=True)
        pk.packkv_encode_block(cache, to_dev(k), to_dev(v), nb)
        oc = O.OracleCache(1, 1, nb, bits, key)
        oc.encode_blocks(k, v, nb)
        compare_encoder(cache, oc)
        assert pk.packkv_get_status(cache) == 0
