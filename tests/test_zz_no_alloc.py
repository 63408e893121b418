"""GPU test of packkv_pv_gemv_noalloc, the p·V entry point that allocates
nothing (for callers that cannot allocate device memory: runtimes that plan all
device memory up front, hosts with no device allocator to pass in, decode loops
that must not trigger the implicit synchronisation of cudaMalloc).

It must give the results of packkv_pv_gemv (within the parity tolerance, 1e-3 of
the sum of |terms| per element) on two calls in a row, work in a fresh process
(its first call sets up the scratch address) as well as after other tests, and
refuse a call that needs more than its fixed scratch.  This file is collected
last so that a run stopping at its first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import oracle as O
from decode_gemv_packkv_b200 import synth
from parity_util import assert_within_terms, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


@pytest.mark.parametrize("bits,group,structured", [(4, 1, False), (2, 4, True), (3, 2, False)])
def test_noalloc_matches_pv_gemv_twice(pk, bits, group, structured):
    B, H = 2, 3
    k, v, q = synth.small_case(900 + bits, B, H, group, 6 * 128 + 51, structured=structured)
    cache = pk.PackKVCache(B, H, 8, bits)
    pk.prefill(cache, to_dev(k), to_dev(v))
    oc = O.OracleCache(B, H, 8, bits)
    oc.encode_blocks(k[:, :, :768], v[:, :, :768], 6)
    for t in range(768, k.shape[2]):
        oc.append_token(k[:, :, t], v[:, :, t])
    T = cache.tokens
    ld = (T + 3) // 4 * 4
    rng = np.random.default_rng(bits)
    for call in range(2):
        p = rng.standard_normal((B, H * group, T)).astype(np.float32)
        pd = torch.zeros((B, H * group, ld), device="cuda")
        pd[:, :, :T] = to_dev(p)
        ref = torch.zeros((B, H * group, 128), device="cuda")
        got = torch.full((B, H * group, 128), 9.0, device="cuda")
        pk.packkv_pv_gemv(cache, pd, ref)
        pk.packkv_pv_gemv_noalloc(cache, pd, got)
        torch.cuda.synchronize()
        _, terms = O.cache_pv(oc, p)
        assert_within_terms(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), terms,
                            f"noalloc vs pv_gemv, call {call}")
    assert pk.packkv_get_status(cache) == 0


def test_noalloc_refuses_more_than_its_scratch(pk):
    """batch*kv_heads = 2048 pairs with G = 8 needs more than the fixed scratch."""
    B, H, G = 64, 32, 8
    cache = pk.PackKVCache(B, H, 1, 4)
    tok = torch.zeros((B, H, 128), dtype=torch.float16, device="cuda")
    pk.packkv_append_token(cache, tok, tok)
    p = torch.zeros((B, H * G, 4), device="cuda")
    out = torch.zeros((B, H * G, 128), device="cuda")
    with pytest.raises(pk.PackKVError) as err:
        pk.packkv_pv_gemv_noalloc(cache, p, out)
    assert err.value.status == pk.ERR_CAPACITY
    assert pk.packkv_pv_noalloc_scratch_bytes() == 8 << 20
