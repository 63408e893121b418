"""GPU parity of ragged batches and block tables against the CPU oracle.

A ragged batch gives every sequence its own length and a block table maps each
sequence's logical blocks to physical ones (the visualisation page, "Read the
caveat": paging and multi-request scheduling).  Checked through the C ABI:
records written by ragged prefills and masked appends are bit-exact at their
physical index entries, and q·Kᵀ, p·V and the fused attention of every sequence
are within 1e-3 * sum|terms| of the oracle's ragged products, with and without
a block table that shares and permutes blocks, and with an empty sequence.
"""
import numpy as np
import pytest
import torch

import oracle as O
from decode_gemv_packkv_b200 import synth
from parity_util import assert_within_terms, gpu_record, gpu_records, to_dev

pytestmark = pytest.mark.gpu

SCALE = 1.0 / np.sqrt(128.0)


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


def _grow(pk, B, H, mb, bits, nb0, appends, seed, structured, key=O.KEY_K_SUM):
    """A ragged GPU cache and its oracle: nb0 blocks for every sequence, then masked
    appends, sequence b taking appends[b] tokens (all starting together)."""
    T = nb0 * 128 + max(appends)
    k, v, _ = synth.small_case(seed, B, H, 1, T, structured=structured)
    cache = pk.PackKVCache(B, H, mb, bits, reorder_key=key, ragged=True, keep_perm=True)
    oc = O.RaggedOracleCache(B, H, mb, bits, key)
    if nb0:
        pk.packkv_encode_block(cache, to_dev(k[:, :, :nb0 * 128].copy()), to_dev(v[:, :, :nb0 * 128].copy()), nb0)
        oc.encode_blocks_ragged(k[:, :, :nb0 * 128], v[:, :, :nb0 * 128], nb0)
    kd, vd = to_dev(k), to_dev(v)
    for s in range(max(appends)):
        active = [b for b in range(B) if s < appends[b]]
        t = nb0 * 128 + s
        pk.packkv_append_token_masked(cache, kd[:, :, t].contiguous(), vd[:, :, t].contiguous(),
                                      [b in active for b in range(B)])
        oc.append_token_ragged(k[:, :, t], v[:, :, t], active)
    assert cache.seq_blocks == oc.seq_blocks and cache.seq_tail == oc.seq_tail
    return cache, oc


def _compare_records(pk, cache, oc):
    for which in ("k", "v"):
        arena, index = gpu_records(cache, which)
        for b in range(oc.batch):
            for h in range(oc.kv_heads):
                for j in range(oc.seq_blocks[b]):
                    rb, jb = oc.physical(b, j)
                    assert gpu_record(arena, index, rb, h, jb) == oc.record(which, rb, h, jb), (which, b, h, j)
    perm = cache.perm.cpu().numpy()
    for b in range(oc.batch):
        for h in range(oc.kv_heads):
            for j in range(oc.seq_blocks[b]):
                rb, jb = oc.physical(b, j)
                assert np.array_equal(perm[rb, h, jb], oc.perm[rb, h, jb])


def _products(pk, cache, oc, G, seed):
    B, H = oc.batch, oc.kv_heads
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    T = max(oc.tokens, 1)
    ld = (T + 3) // 4 * 4
    scores = torch.full((B, H * G, ld), 7.0, device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    ref, terms = O.ragged_qk(oc, q, SCALE)
    s_np = scores.cpu().numpy()
    for b in range(B):
        Tb = oc.seq_tokens(b)
        assert_within_terms(s_np[b, :, :Tb], ref[b, :, :Tb], terms[b, :, :Tb], f"scores of sequence {b}")
        assert np.all(s_np[b, :, Tb:] == 7.0), f"sequence {b}: written past its length"
    p = rng.standard_normal((B, H * G, ld)).astype(np.float32)
    out = torch.full((B, H * G, 128), 7.0, device="cuda")
    pk.packkv_pv_gemv(cache, to_dev(p), out)
    ref, terms = O.ragged_pv(oc, p)
    assert_within_terms(out.cpu().numpy(), ref, terms, "p·V")
    att = torch.full((B, H * G, 128), 7.0, device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, att)
    ref, terms = O.ragged_attention(oc, q, SCALE)
    assert_within_terms(att.cpu().numpy(), ref, terms, "attention")
    assert pk.packkv_get_status(cache) == 0


@pytest.mark.parametrize("bits,G,structured", [(4, 1, False), (2, 4, True), (3, 2, True)])
def test_ragged_growth_and_products(pk, bits, G, structured):
    """Sequences growing by different amounts across block boundaries."""
    cache, oc = _grow(pk, 3, 2, 6, bits, 2, [300, 90, 1], 800 + bits, structured)
    assert [oc.seq_tokens(b) for b in range(3)] == [556, 346, 257]
    _compare_records(pk, cache, oc)
    _products(pk, cache, oc, G, bits)


def test_block_table_shares_and_permutes_blocks(pk):
    """After growth, a block table points sequence 2's two blocks at sequence 0's
    first two (a shared prompt) and reverses sequence 0's three blocks; the products
    read through it."""
    B, H, mb, bits = 3, 2, 6, 4
    cache, oc = _grow(pk, B, H, mb, bits, 2, [300, 90, 1], 71, True)
    table = np.arange(B * mb, dtype=np.int32).reshape(B, mb)
    table[2, 0], table[2, 1] = 0, 1
    table[0, :3] = [2, 1, 0]
    oc.table = table.astype(np.int64)
    oc._decoded.clear()
    cache.block_table = torch.from_numpy(table).cuda()
    cache.s.block_table = cache.block_table.data_ptr()
    _products(pk, cache, oc, 2, 5)


def test_ragged_empty_sequence_and_uniform_table(pk):
    """A sequence that never took a token gets zero outputs and no scores; a uniform
    cache with a block table reads through the table."""
    cache, oc = _grow(pk, 3, 2, 3, 3, 0, [140, 60, 0], 91, False)
    assert oc.seq_tokens(2) == 0
    _products(pk, cache, oc, 1, 3)
    # uniform cache, table swapping the two blocks of every sequence
    B, H = 2, 2
    k, v, q = synth.small_case(92, B, H, 2, 2 * 128 + 33)
    table = np.tile(np.array([1, 0, 2], np.int32), (B, 1)) + 3 * np.arange(B, dtype=np.int32)[:, None]
    ucache = pk.PackKVCache(B, H, 3, 4)
    pk.prefill(ucache, to_dev(k), to_dev(v))
    ucache.block_table = torch.from_numpy(table).cuda()
    ucache.s.block_table = ucache.block_table.data_ptr()
    uo = O.OracleCache(B, H, 3, 4)
    uo.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, k.shape[2]):
        uo.append_token(k[:, :, t], v[:, :, t])
    ro = O.RaggedOracleCache(B, H, 3, 4, table=table)
    ro.k_arena, ro.v_arena, ro.k_index, ro.v_index = uo.k_arena, uo.v_arena, uo.k_index, uo.v_index
    ro.k_tail, ro.v_tail = uo.k_tail, uo.v_tail
    ro.seq_blocks, ro.seq_tail = [2] * B, [33] * B
    ld = (ro.tokens + 3) // 4 * 4
    scores = torch.zeros((B, H * 2, ld), device="cuda")
    pk.packkv_qk_gemv(ucache, to_dev(q), SCALE, scores)
    ref, terms = O.ragged_qk(ro, q, SCALE)
    assert_within_terms(scores.cpu().numpy()[:, :, :ro.tokens], ref, terms, "scores through a block table")


def test_ragged_many_sequences(pk, monkeypatch):
    """512 sequences of 4 KV heads, lengths from 1 to 1200 tokens: about 12k items,
    several per warp, so warps cross many sequence boundaries of unequal length and
    ragged tails.  Every sequence is checked.  The tokens of every sequence are drawn
    from four distinct 128-token blocks, so the oracle encodes and decodes each
    distinct block once (memoised by content)."""
    import functools

    import oracle.packkv_oracle as OM
    B, H, bits = 512, 4, 4
    real_enc, real_parse = OM.encode_block, OM.parse_record
    enc = functools.lru_cache(maxsize=None)(lambda kb, vb, b_, key, mode: real_enc(
        np.frombuffer(kb, np.float16).reshape(128, 128), np.frombuffer(vb, np.float16).reshape(128, 128), b_, key,
        mode))
    monkeypatch.setattr(OM, "encode_block", lambda k_, v_, b_, key=O.KEY_K_SUM, mode=O.UNITS_FOR: enc(
        np.ascontiguousarray(k_, np.float16).tobytes(), np.ascontiguousarray(v_, np.float16).tobytes(), b_, key,
        mode))
    monkeypatch.setattr(OM, "parse_record", functools.lru_cache(maxsize=None)(real_parse))
    pool_k, pool_v, _ = synth.small_case(94, 1, 4, 1, 128)
    rng = np.random.default_rng(4)
    lens = rng.integers(1, 1200, B)
    T = int(lens.max())
    t = np.arange(T)
    which = (np.arange(B)[:, None] + t[None, :] // 128) % 4              # pool block of (sequence, token)
    k = pool_k[0, which, t[None, :] % 128]                               # [B, T, 128]
    v = pool_v[0, which, t[None, :] % 128]
    k = np.ascontiguousarray(np.repeat(k[:, None], H, axis=1))           # every head alike
    v = np.ascontiguousarray(np.repeat(v[:, None], H, axis=1))
    cache = pk.PackKVCache(B, H, 10, bits, ragged=True, keep_perm=True)
    oc = O.RaggedOracleCache(B, H, 10, bits)
    kd, vd = to_dev(k), to_dev(v)
    for s_ in range(T):
        active = lens > s_
        pk.packkv_append_token_masked(cache, kd[:, :, s_].contiguous(), vd[:, :, s_].contiguous(), list(active))
        oc.append_token_ragged(k[:, :, s_], v[:, :, s_], list(np.nonzero(active)[0]))
    assert cache.seq_blocks == oc.seq_blocks and cache.seq_tail == oc.seq_tail
    _compare_records(pk, cache, oc)
    _products(pk, cache, oc, 1, 6)
