"""GPU parity of the fused decode attention (packkv_attention_decode) against the
CPU oracle's softmax(scale q·K̂ᵀ)·V̂ over the packed cache.

Tolerance: every output element within 1e-3 of the sum over tokens of
|p_i * v_hat_ic| (the oracle's terms, with the exact fp64 softmax).  Small cases
span several blocks, pack groups and ragged tails, compressed and raw records;
the full 32-head 32k-token cache is checked on one whole sequence in the launch
configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import oracle as O
from decode_gemv_packkv_b200 import synth
from parity_util import assert_within_terms, to_dev

pytestmark = pytest.mark.gpu

SCALE = 1.0 / np.sqrt(128.0)


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


def _build(pk, k, v, bits):
    B, H, T, _ = k.shape
    nb = T // 128
    cache = pk.PackKVCache(B, H, nb + 1, bits)
    pk.prefill(cache, to_dev(k), to_dev(v))
    ocache = O.OracleCache(B, H, nb + 1, bits)
    ocache.encode_blocks(k[:, :, :nb * 128], v[:, :, :nb * 128], nb)
    for t in range(nb * 128, T):
        ocache.append_token(k[:, :, t], v[:, :, t])
    return cache, ocache


def _attn(pk, cache, q, scale=SCALE):
    B, Hq, _ = q.shape
    out = torch.full((B, Hq, 128), 7.0, dtype=torch.float32, device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), scale, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("structured", [False, True])
def test_attention_parity(pk, bits, group, structured):
    tail = {1: 0, 2: 37, 4: 127, 8: 1}[group]
    k, v, q = synth.small_case(500 + bits * 10 + group, 2, 2, group, 3 * 128 + tail, structured=structured)
    cache, ocache = _build(pk, k, v, bits)
    got = _attn(pk, cache, q)
    ref, terms = O.cache_attention(ocache, q, SCALE)
    assert_within_terms(got, ref, terms, "attention")
    assert pk.packkv_get_status(cache) == 0


def test_attention_tail_only_and_large_scores(pk):
    """Only tail tokens (no block), and a large scale: a sharply peaked softmax."""
    k, v, q = synth.small_case(61, 1, 2, 2, 77)
    cache, ocache = _build(pk, k, v, 4)
    assert cache.n_blocks == 0 and cache.tail_len == 77
    for scale in (SCALE, 4.0):
        got = _attn(pk, cache, q, scale)
        ref, terms = O.cache_attention(ocache, q, scale)
        assert_within_terms(got, ref, terms, f"tail-only attention, scale {scale}")


@pytest.mark.parametrize("bits", [2, 4])
def test_attention_peaked_softmax_over_blocks(pk, bits):
    """A large scale over several blocks: most probabilities underflow to zero, so whole
    records see p = 0 (zero digit tables) next to records that carry all the weight."""
    k, v, q = synth.small_case(65 + bits, 1, 2, 4, 5 * 128 + 19)
    cache, ocache = _build(pk, k, v, bits)
    got = _attn(pk, cache, q, 4.0)
    ref, terms = O.cache_attention(ocache, q, 4.0)
    assert_within_terms(got, ref, terms, "peaked attention")
    assert pk.packkv_get_status(cache) == 0


def test_attention_many_items_per_warp_and_determinism(pk):
    """A long sequence over few (sequence, head) pairs: every warp spans several
    records and (sequence, head) boundaries; two calls agree bit for bit, also with
    a dirty workspace."""
    k, v, q = synth.small_case(62, 1, 2, 4, 40 * 128 + 9)
    cache, ocache = _build(pk, k, v, 4)
    a = _attn(pk, cache, q)
    cache.attention_workspace(8).fill_(0xCD)
    b = _attn(pk, cache, q)
    assert np.array_equal(a, b)
    ref, terms = O.cache_attention(ocache, q, SCALE)
    assert_within_terms(a, ref, terms, "long attention")


def test_attention_streaming_growth(pk):
    """After token-by-token growth across a block boundary the fused result follows."""
    B, H, G = 1, 2, 2
    k, v, q = synth.small_case(63, B, H, G, 128 + 150)
    cache = pk.PackKVCache(B, H, 4, 4)
    ocache = O.OracleCache(B, H, 4, 4)
    pk.packkv_encode_block(cache, to_dev(k[:, :, :128].copy()), to_dev(v[:, :, :128].copy()), 1)
    ocache.encode_blocks(k[:, :, :128], v[:, :, :128], 1)
    for t in range(128, k.shape[2]):
        pk.packkv_append_token(cache, to_dev(k[:, :, t].copy()), to_dev(v[:, :, t].copy()))
        ocache.append_token(k[:, :, t], v[:, :, t])
        if t in (128, 200, 255, 256, k.shape[2] - 1):
            got = _attn(pk, cache, q)
            ref, terms = O.cache_attention(ocache, q, SCALE)
            assert_within_terms(got, ref, terms, f"attention after token {t}")


def test_attention_equals_separate_products(pk):
    """The fused pass and q·Kᵀ, softmax, p·V through the separate calls agree within
    the tolerance (they decode the same records)."""
    k, v, q = synth.small_case(64, 2, 2, 2, 6 * 128 + 33)
    cache, ocache = _build(pk, k, v, 4)
    got = _attn(pk, cache, q)
    T = cache.tokens
    ld = (T + 3) // 4 * 4
    scores = torch.zeros((2, 4, ld), device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    p = torch.zeros_like(scores)
    p[:, :, :T] = torch.softmax(scores[:, :, :T], dim=-1)
    out = torch.zeros((2, 4, 128), device="cuda")
    pk.packkv_pv_gemv(cache, p, out)
    _, terms = O.cache_attention(ocache, q, SCALE)
    assert_within_terms(got, out.cpu().numpy().astype(np.float64), terms, "fused vs separate")


def test_attention_rejects_an_empty_cache(pk):
    cache = pk.PackKVCache(1, 1, 2, 4)
    out = torch.zeros((1, 1, 128), device="cuda")
    with pytest.raises(pk.PackKVError) as err:
        pk.packkv_attention_decode(cache, torch.zeros((1, 1, 128), dtype=torch.float16, device="cuda"), 1.0, out)
    assert err.value.status == pk.ERR_INVALID_ARG


@pytest.mark.parametrize("wid,bits,h", [(1, 4, 5), (2, 2, 3)])
def test_attention_full_workload_one_sequence(pk, wid, bits, h):
    """Full-size caches (32-head 32k-token 4-bit; 8 KV heads x 4 query heads, 131k
    tokens, 2-bit): one whole (sequence, KV head) against the oracle, in the launch
    configuration the benchmark uses (hundreds of warps merged per output row)."""
    w = synth.WORKLOADS[wid]
    T = w.seq
    G = w.group
    kd = torch.empty((w.batch, w.kv_heads, T, 128), dtype=torch.float16, device="cuda")
    vd = torch.empty_like(kd)
    for b in range(w.batch):
        for hh in range(w.kv_heads):
            ks, vs = synth.kv_slice(w.seed, w.kv_heads, b, hh, T)
            kd[b, hh].copy_(torch.from_numpy(ks))
            vd[b, hh].copy_(torch.from_numpy(vs))
    cache = pk.PackKVCache(w.batch, w.kv_heads, T // 128, bits)
    pk.packkv_encode_block(cache, kd, vd, T // 128)
    q = synth.queries(w, 0)
    out = torch.zeros((w.batch, w.q_heads, 128), device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, out)
    got = out.cpu().numpy()
    oc = O.OracleCache(1, 1, T // 128, bits)
    oc.encode_blocks(kd[0:1, h:h + 1].cpu().numpy(), vd[0:1, h:h + 1].cpu().numpy(), T // 128)
    ref, terms = O.cache_attention(oc, q[0:1, h * G:(h + 1) * G], SCALE)
    assert_within_terms(got[0:1, h * G:(h + 1) * G], ref, terms, f"full-size attention, kv head {h}")
    assert np.all(np.isfinite(got))
