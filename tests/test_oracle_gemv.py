"""Pins for the oracle's decode products (CPU only).

q·Kᵀ and p·V over the packed cache (PackKV paper page, Figure 1 attention at
decode, Figure 2 fused decompression + matrix-vector product), and the
permutation invariance that licenses the reorder (TL;DR; visualisation page,
"Permutation invariance, visually").
"""
import itertools

import numpy as np
import pytest

import oracle as O
from decode_gemv_packkv_b200 import synth


def _grid_kv(rng, B, H, T, bits):
    """K exactly on a per-(block, channel) grid and V on a per-token grid, so the
    quantizer is lossless and the decoded cache equals the input exactly."""
    qmax = (1 << bits) - 1
    nk = rng.integers(0, qmax + 1, (B, H, T, 128))
    nv = rng.integers(0, qmax + 1, (B, H, T, 128))
    nk[:, :, ::128, :] = 0
    nk[:, :, 1::128, :] = qmax           # every block spans the full code range per channel
    nv[..., 0], nv[..., 1] = 0, qmax     # every token spans it too
    ek = rng.integers(-4, 2, (B, H, T // 128, 1, 128)).repeat(128, axis=3).reshape(B, H, T, 128)
    mk = np.round(rng.uniform(-4, 4, (B, H, T // 128, 1, 128)) * 16).repeat(128, axis=3).reshape(B, H, T, 128) / 16
    ev = rng.integers(-4, 2, (B, H, T, 1))
    mv = np.round(rng.uniform(-4, 4, (B, H, T, 1)) * 16) / 16
    k = (mk + np.exp2(ek) * nk)
    v = (mv + np.exp2(ev) * nv)
    assert np.array_equal(k.astype(np.float16).astype(np.float64), k)
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
    return k.astype(np.float16), v.astype(np.float16)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_products_on_grid_inputs_match_plain_attention_algebra(bits):
    """Lossless inputs: scores equal scale * K q in the ORIGINAL token order after
    undoing the storage permutation; p·V equals the plain weighted sum of V."""
    rng = np.random.default_rng(100 + bits)
    B, H, G, T = 2, 2, 2, 256 + 40
    k, v = _grid_kv(rng, B, H, 384, bits)
    k, v = k[:, :, :T], v[:, :, :T]
    q = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    cache = O.OracleCache(B, H, 4, bits)
    cache.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, T):
        cache.append_token(k[:, :, t], v[:, :, t])
    scale = 1 / np.sqrt(128)
    scores, sums = O.cache_qk(cache, q, scale)
    p = rng.random((B, H * G, T))
    out, _ = O.cache_pv(cache, p)
    for b in range(B):
        for h in range(H):
            # storage position -> original token index
            pos = np.concatenate([256 * 0 + 128 * i + cache.perm[b, h, i].astype(np.int64)
                                  for i in range(2)] + [np.arange(256, T)])
            kk = k[b, h].astype(np.float64)
            vv = v[b, h].astype(np.float64)
            for g in range(G):
                hq = h * G + g
                want = scale * (kk @ q[b, hq].astype(np.float64))
                np.testing.assert_allclose(scores[b, hq], want[pos], rtol=1e-12, atol=1e-12)
                # p given in storage order multiplies the token stored there
                want_o = (p[b, hq][:, None] * vv[pos]).sum(axis=0)
                np.testing.assert_allclose(out[b, hq], want_o, rtol=1e-12, atol=1e-12)
    assert np.all(sums >= np.abs(scores) - 1e-12)


def test_one_hot_query_extracts_a_decoded_channel():
    k, v, _ = synth.small_case(3, 1, 1, 1, 128)
    cache = O.OracleCache(1, 1, 1, 4)
    cache.encode_blocks(k, v, 1)
    rec = O.parse_record(cache.record("k", 0, 0, 0))
    for c in (0, 17, 127):
        q = np.zeros((1, 1, 128), np.float16)
        q[0, 0, c] = 1
        s, _ = O.cache_qk(cache, q, 1.0)
        np.testing.assert_array_equal(s[0, 0], rec.mn[c].astype(np.float64)
                                      + rec.scale[c].astype(np.float64) * rec.codes[:, c])


def test_one_hot_p_extracts_a_decoded_token():
    k, v, _ = synth.small_case(4, 1, 1, 1, 128)
    cache = O.OracleCache(1, 1, 1, 3)
    cache.encode_blocks(k, v, 1)
    rec = O.parse_record(cache.record("v", 0, 0, 0))
    for r in (0, 63, 127):
        p = np.zeros((1, 1, 128))
        p[0, 0, r] = 1
        o, _ = O.cache_pv(cache, p)
        np.testing.assert_array_equal(o[0, 0], rec.mn[r].astype(np.float64)
                                      + rec.scale[r].astype(np.float64) * rec.codes[r])


def test_attention_permutation_invariance_brute_force():
    """All 5040 joint permutations of 7 (K, V) pairs leave attention unchanged."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal(4)
    k = rng.standard_normal((7, 4))
    v = rng.standard_normal((7, 4))
    ref = O.attention(q, k, v, 0.5)
    mag = np.abs(v).sum(axis=0)
    for perm in itertools.permutations(range(7)):
        got = O.attention(q, k[list(perm)], v[list(perm)], 0.5)
        assert np.all(np.abs(got - ref) <= 1e-12 * mag)
    # a permutation applied to K alone does change it (the binding matters)
    bad = O.attention(q, k[[1, 0, 2, 3, 4, 5, 6]], v, 0.5)
    assert np.max(np.abs(bad - ref)) > 1e-6


def test_attention_over_packed_cache_equals_unpermuted_attention():
    """Block scale: softmax over storage-order scores, then p·V in storage order,
    equals fp64 attention over the decoded cache put back in token order."""
    k, v, q = synth.small_case(8, 1, 2, 2, 384 + 50, structured=True)
    cache = O.OracleCache(1, 2, 4, 4)
    cache.encode_blocks(k[:, :, :384], v[:, :, :384], 3)
    for t in range(384, 434):
        cache.append_token(k[:, :, t], v[:, :, t])
    scale = 1 / np.sqrt(128)
    scores, _ = O.cache_qk(cache, q, scale)
    out, _ = O.cache_pv(cache, O.softmax(scores))
    for h in range(2):
        kd, vd = cache.decoded("k", 0, h), cache.decoded("v", 0, h)
        pos = np.concatenate([128 * i + cache.perm[0, h, i].astype(np.int64) for i in range(3)]
                             + [np.arange(384, 434)])
        k_tok = np.empty_like(kd)
        v_tok = np.empty_like(vd)
        k_tok[pos], v_tok[pos] = kd, vd
        for g in range(2):
            want = O.attention(q[0, 2 * h + g].astype(np.float64), k_tok, v_tok, scale)
            np.testing.assert_allclose(out[0, 2 * h + g], want, rtol=1e-12, atol=1e-12)


def test_quantization_error_propagates_within_bound():
    """|scores(decoded) - scores(original)| <= scale * sum_c |q_c| * bound_c."""
    k, v, q = synth.small_case(21, 1, 1, 1, 128)
    for bits in (2, 3, 4):
        cache = O.OracleCache(1, 1, 1, bits)
        cache.encode_blocks(k, v, 1)
        s, _ = O.cache_qk(cache, q, 1.0)
        rec = O.parse_record(cache.record("k", 0, 0, 0))
        exact = (k[0, 0].astype(np.float64) @ q[0, 0].astype(np.float64))[cache.perm[0, 0, 0]]
        bound = np.abs(q[0, 0].astype(np.float64)) @ O.quant_error_bound(rec.scale, bits)
        assert np.all(np.abs(s[0, 0] - exact) <= bound)


@pytest.mark.parametrize("bits", [2, 4])
def test_fused_attention_on_grid_inputs_is_plain_softmax_attention(bits):
    """Lossless inputs: the oracle's decode attention over the packed, permuted cache
    equals textbook softmax attention (numpy, fp64) over the original tokens in
    arrival order: the storage permutation and the packing drop out."""
    rng = np.random.default_rng(200 + bits)
    B, H, G, T = 1, 2, 2, 256 + 17
    k, v = _grid_kv(rng, B, H, 384, bits)
    k, v = k[:, :, :T], v[:, :, :T]
    q = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    cache = O.OracleCache(B, H, 4, bits)
    cache.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, T):
        cache.append_token(k[:, :, t], v[:, :, t])
    scale = 1 / np.sqrt(128)
    out, terms = O.cache_attention(cache, q, scale)
    for b in range(B):
        for h in range(H):
            kk = k[b, h].astype(np.float64)
            vv = v[b, h].astype(np.float64)
            for g in range(G):
                hq = h * G + g
                s = scale * (kk @ q[b, hq].astype(np.float64))
                e = np.exp(s - s.max())
                want = (e / e.sum()) @ vv
                np.testing.assert_allclose(out[b, hq], want, rtol=1e-10, atol=1e-10)
                # the tolerance scale bounds the result (triangle inequality) and is the
                # probability-weighted sum of |v|
                assert np.all(terms[b, hq] >= np.abs(out[b, hq]) - 1e-12)
                np.testing.assert_allclose(terms[b, hq], (e / e.sum()) @ np.abs(vv), rtol=1e-10)


def test_fused_attention_probabilities_sum_to_one():
    """With V constant 1 in every channel the output is the sum of the probabilities: 1."""
    k, _, q = synth.small_case(7, 1, 1, 2, 128 * 2 + 5)
    v = np.ones_like(k)
    cache = O.OracleCache(1, 1, 3, 4)
    cache.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, k.shape[2]):
        cache.append_token(k[:, :, t], v[:, :, t])
    out, _ = O.cache_attention(cache, q, 0.3)
    np.testing.assert_allclose(out, 1.0, rtol=1e-12)
