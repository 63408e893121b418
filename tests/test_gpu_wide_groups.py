"""GPU parity for wide query groups: 16, 32 and 64 query heads per KV head.

A wide group arises from models whose query heads far outnumber their KV heads
and from decoding several queries per KV head in one step (speculative
decoding: S draft positions x G heads share the kv head's cache).  The library
serves such groups in launches of 8 query heads.  Checked through the C ABI
against the CPU oracle (1e-3 * sum|terms| per element): q·Kᵀ, p·V and the fused
attention, on raw and compressed records, with ragged tails.
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


@pytest.mark.parametrize("bits,group,structured", [(4, 16, False), (2, 32, True), (3, 64, False), (4, 16, True)])
def test_wide_group_parity(pk, bits, group, structured):
    B, H = 2, 2
    k, v, q = synth.small_case(600 + bits + group, B, H, group, 3 * 128 + 45, structured=structured)
    cache = pk.PackKVCache(B, H, 4, bits)
    pk.prefill(cache, to_dev(k), to_dev(v))
    oc = O.OracleCache(B, H, 4, bits)
    oc.encode_blocks(k[:, :, :384], v[:, :, :384], 3)
    for t in range(384, k.shape[2]):
        oc.append_token(k[:, :, t], v[:, :, t])
    T = cache.tokens
    ld = (T + 3) // 4 * 4
    scores = torch.full((B, H * group, ld), 7.0, device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    ref, terms = O.cache_qk(oc, q, SCALE)
    got = scores.cpu().numpy()
    assert_within_terms(got[:, :, :T], ref, terms, f"scores, G={group}")
    assert np.all(got[:, :, T:] == 7.0)
    p = O.softmax(ref).astype(np.float32)
    pd = torch.zeros((B, H * group, ld), device="cuda")
    pd[:, :, :T] = to_dev(p)
    out = torch.full((B, H * group, 128), 7.0, device="cuda")
    pk.packkv_pv_gemv(cache, pd, out)
    ref_o, terms_o = O.cache_pv(oc, p)
    assert_within_terms(out.cpu().numpy(), ref_o, terms_o, f"p·V, G={group}")
    att = torch.full((B, H * group, 128), 7.0, device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, att)
    ref_a, terms_a = O.cache_attention(oc, q, SCALE)
    assert_within_terms(att.cpu().numpy(), ref_a, terms_a, f"attention, G={group}")
    assert pk.packkv_get_status(cache) == 0


def test_speculative_queries_share_the_cache(pk):
    """S = 4 draft positions of a G = 4 GQA layer read each kv head's cache as a group
    of 16 query rows (position s of head g at row h*16 + s*4 + g): every row matches
    the oracle's attention for its own query vector."""
    B, H, G, S, bits = 1, 2, 4, 4, 4
    k, v, _ = synth.small_case(640, B, H, 1, 2 * 128 + 17)
    q_steps = np.random.default_rng(641).standard_normal((S, B, H * G, 128)).astype(np.float16)
    cache = pk.PackKVCache(B, H, 3, bits)
    pk.prefill(cache, to_dev(k), to_dev(v))
    oc = O.OracleCache(B, H, 3, bits)
    oc.encode_blocks(k[:, :, :256], v[:, :, :256], 2)
    for t in range(256, k.shape[2]):
        oc.append_token(k[:, :, t], v[:, :, t])
    qw = q_steps.reshape(S, B, H, G, 128).transpose(1, 2, 0, 3, 4).reshape(B, H * S * G, 128)
    att = torch.zeros((B, H * S * G, 128), device="cuda")
    pk.packkv_attention_decode(cache, to_dev(np.ascontiguousarray(qw)), SCALE, att)
    wide = att.cpu().numpy().reshape(B, H, S, G, 128)
    for s in range(S):
        ref, terms = O.cache_attention(oc, q_steps[s], SCALE)
        assert_within_terms(wide[:, :, s].reshape(B, H * G, 128), ref, terms, f"draft position {s}")
