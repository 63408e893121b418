"""Pins for the oracle's ragged batches and block table (CPU only).

A ragged batch gives every sequence its own length (the visualisation page,
"Read the caveat": paging and multi-request scheduling).  Its oracle reduces to
the already-pinned uniform one: every sequence of a ragged cache must equal a
one-sequence uniform cache fed the same tokens (records bit for bit, decoded
values, products), and a block table that points one sequence at another's
blocks must decode to exactly those blocks.
"""
import numpy as np
import pytest

import oracle as O
from decode_gemv_packkv_b200 import synth

SCALE = 1.0 / np.sqrt(128.0)


def _streams(B, H, T, seed, structured=False):
    k, v, _ = synth.small_case(seed, B, H, 1, T, structured=structured)
    return k, v


def _uniform_of(k1, v1, T, bits, max_blocks, key=O.KEY_K_SUM):
    """One sequence fed token by token into the uniform oracle cache."""
    u = O.OracleCache(1, k1.shape[0], max_blocks, bits, key)
    for t in range(T):
        u.append_token(k1[None, :, t], v1[None, :, t])
    return u


@pytest.mark.parametrize("bits", [2, 4])
def test_ragged_appends_equal_per_sequence_uniform_caches(bits):
    """Sequences joining at different steps (so their lengths differ) with a shared
    prefill: each one equals its own uniform cache, record for record."""
    B, H, nb0 = 3, 2, 1
    starts = [0, 40, 200]          # step at which sequence b starts appending
    steps = 300
    k, v = _streams(B, H, nb0 * 128 + steps, 77 + bits, structured=(bits == 2))
    r = O.RaggedOracleCache(B, H, 4, bits)
    r.encode_blocks_ragged(k[:, :, :128], v[:, :, :128], nb0)
    pos = [128] * B
    for s in range(steps):
        active = [b for b in range(B) if s >= starts[b]]
        tok_k = np.zeros((B, H, 128), np.float16)
        tok_v = np.zeros_like(tok_k)
        for b in active:
            tok_k[b], tok_v[b] = k[b, :, pos[b]], v[b, :, pos[b]]
            pos[b] += 1
        r.append_token_ragged(tok_k, tok_v, active)
    for b in range(B):
        T = pos[b]
        assert r.seq_tokens(b) == T
        u = _uniform_of(k[b], v[b], T, bits, 4)
        assert (u.n_blocks, u.tail_len) == (r.seq_blocks[b], r.seq_tail[b])
        for h in range(H):
            for j in range(r.seq_blocks[b]):
                rb, jb = r.physical(b, j)
                assert r.record("k", rb, h, jb) == u.record("k", 0, h, j)
                assert r.record("v", rb, h, jb) == u.record("v", 0, h, j)
            assert np.array_equal(r.decoded("k", b, h), u.decoded("k", 0, h))
            assert np.array_equal(r.decoded("v", b, h), u.decoded("v", 0, h))


def test_ragged_arena_order_follows_sequences():
    """An append that completes several tails writes their records in ascending
    (sequence, head) order, one after the other."""
    B, H = 3, 2
    k, v = _streams(B, H, 256, 5)
    r = O.RaggedOracleCache(B, H, 2, 3)
    for t in range(127):
        r.append_token_ragged(k[:, :, t], v[:, :, t], active=[0, 2])
    r.append_token_ragged(k[:, :, 127], v[:, :, 127], active=[0, 2])   # tails of 0 and 2 complete
    offs = [(int(r.k_index[b, h, 0, 0]), int(r.k_index[b, h, 0, 1])) for b in (0, 2) for h in range(H)]
    at = 0
    for off, ln in offs:
        assert off == at
        at += ln
    assert at * 16 == len(r.k_arena)
    assert r.seq_blocks == [1, 0, 1] and r.seq_tail == [0, 0, 0]


def test_block_table_shares_a_prefix():
    """Sequence 1's first two logical blocks point at sequence 0's physical blocks (a
    common prompt): it decodes to those blocks followed by its own block and tail, and
    its scores and outputs are the plain products over that concatenation."""
    B, H, mb, bits = 2, 2, 4, 4
    table = np.arange(B * mb).reshape(B, mb)
    table[1, 0], table[1, 1] = table[0, 0], table[0, 1]
    table[1, 2] = 1 * mb + 0            # its third logical block in its own first physical slot
    k, v = _streams(B, H, 3 * 128 + 50, 31)
    r = O.RaggedOracleCache(B, H, mb, bits, table=table)
    # sequence 0: 2 blocks + a 10-token tail; sequence 1 reuses those 2 blocks
    r.encode_blocks_ragged(k[:1, :, :256].repeat(2, 0), v[:1, :, :256].repeat(2, 0), 2)
    assert r.record("k", 0, 0, 0) == r.record("k", 0, 0, 0)
    for t in range(256, 256 + 128 + 20):
        active = [1] if t < 256 + 128 else [0, 1]
        r.append_token_ragged(k[:, :, t], v[:, :, t], active)
    assert r.seq_blocks == [2, 3] and r.seq_tail == [20, 20]
    for h in range(H):
        d0, d1 = r.decoded("k", 0, h), r.decoded("k", 1, h)
        assert np.array_equal(d1[:256], d0[:256])
        own = O.OracleCache(1, H, 1, bits)
        own.encode_blocks(k[1:, :, 256:384], v[1:, :, 256:384], 1)
        assert np.array_equal(d1[256:384], own.decoded("k", 0, h)[:128])
        assert np.array_equal(d1[384:], k[1, h, 384:404].astype(np.float64))
    q = np.random.default_rng(0).standard_normal((B, H * 2, 128)).astype(np.float16)
    s, terms = O.ragged_qk(r, q, SCALE)
    for b in range(B):
        for h in range(H):
            want, wterms = O.qk_scores(q[b, 2 * h:2 * h + 2], r.decoded("k", b, h), SCALE)
            Tb = r.seq_tokens(b)
            assert np.array_equal(s[b, 2 * h:2 * h + 2, :Tb], want)
            assert np.all(np.isnan(s[b, :, Tb:]))


def test_ragged_products_reduce_to_uniform_products():
    """ragged_qk / ragged_pv / ragged_attention of each sequence equal the uniform
    cache_qk / cache_pv / cache_attention of that sequence alone."""
    B, H, G, bits = 3, 2, 2, 3
    lens = [128 + 7, 3 * 128, 2 * 128 + 100]
    k, v = _streams(B, H, max(lens), 19, structured=True)
    r = O.RaggedOracleCache(B, H, 4, bits)
    pos = [0] * B
    for t in range(max(lens)):
        active = [b for b in range(B) if pos[b] < lens[b]]
        r.append_token_ragged(k[:, :, t], v[:, :, t], active)
        for b in active:
            pos[b] += 1
    q = np.random.default_rng(1).standard_normal((B, H * G, 128)).astype(np.float16)
    s, _ = O.ragged_qk(r, q, SCALE)
    p = np.random.default_rng(2).random((B, H * G, max(lens))).astype(np.float32)
    o, _ = O.ragged_pv(r, p)
    a, _ = O.ragged_attention(r, q, SCALE)
    for b in range(B):
        u = _uniform_of(k[b], v[b], lens[b], bits, 4)
        us, _ = O.cache_qk(u, q[b:b + 1], SCALE)
        assert np.array_equal(s[b:b + 1, :, :lens[b]], us)
        uo, _ = O.cache_pv(u, p[b:b + 1, :, :lens[b]])
        assert np.array_equal(o[b:b + 1], uo)
        ua, _ = O.cache_attention(u, q[b:b + 1], SCALE)
        assert np.allclose(a[b:b + 1], ua, rtol=0, atol=1e-12)


def test_empty_sequence_attends_to_nothing():
    """A sequence that never took a token has zero attention output (an empty softmax
    weights nothing); the other sequences are unaffected."""
    B, H, bits = 2, 2, 4
    k, v = _streams(B, H, 140, 23)
    r = O.RaggedOracleCache(B, H, 2, bits)
    for t in range(140):
        r.append_token_ragged(k[:, :, t], v[:, :, t], active=[0])
    assert r.seq_tokens(1) == 0
    q = np.random.default_rng(3).standard_normal((B, H, 128)).astype(np.float16)
    a, terms = O.ragged_attention(r, q, SCALE)
    assert np.array_equal(a[1], np.zeros((H, 128))) and np.array_equal(terms[1], np.zeros((H, 128)))
    u = _uniform_of(k[0], v[0], 140, bits, 2)
    ua, _ = O.cache_attention(u, q[:1], SCALE)
    assert np.allclose(a[:1], ua, rtol=0, atol=1e-12)
