"""GPU tests of packkv_pv_gemv_noalloc, the p·V entry point that allocates nothing.

It exists for callers that cannot allocate device memory: runtimes that plan
all device memory up front and forbid later allocations, C or foreign-function
hosts that have no device allocator to hand the library, and decode loops that
must not trigger the implicit device synchronisation of cudaMalloc.  Its
split-K partials live in the library's own fixed 8 MiB device array.

Checked here, through the C ABI: on two calls in a row its output matches both
packkv_pv_gemv's and the CPU oracle's (1e-3 of the sum of |terms| per element,
the tolerance of every parity test); its very first call in a fresh process
(which looks up the array's device address) is right; T == 0 gives zeros; and at
the capacity limit the largest call that fits runs correctly while one more
(sequence, head) pair is refused with PACKKV_ERR_CAPACITY before any launch.
This file is collected last, so a run that stops at its first failure has run
every other test.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle as O
from decode_gemv_packkv_b200 import synth
from parity_util import assert_within_terms, to_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


@pytest.mark.parametrize("bits,group,structured", [(4, 1, False), (2, 4, True), (3, 2, False), (4, 8, True)])
def test_noalloc_matches_pv_gemv_and_oracle_twice(pk, bits, group, structured):
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
        want, terms = O.cache_pv(oc, p)
        assert_within_terms(got.cpu().numpy(), want, terms, f"noalloc vs oracle, call {call}")
        assert_within_terms(got.cpu().numpy(), ref.cpu().numpy().astype(np.float64), terms,
                            f"noalloc vs packkv_pv_gemv, call {call}")
    assert pk.packkv_get_status(cache) == 0


def test_noalloc_empty_cache_gives_zeros(pk):
    cache = pk.PackKVCache(2, 2, 4, 3)
    out = torch.full((2, 4, 128), 5.0, device="cuda")
    pk.packkv_pv_gemv_noalloc(cache, torch.zeros((2, 4, 4), device="cuda"), out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def _tail_only_cache(pk, pairs, G, seed):
    """A cache of `pairs` sequences x 1 KV head holding one appended token each."""
    cache = pk.PackKVCache(pairs, 1, 1, 4, arena_bytes=16)
    rng = np.random.default_rng(seed)
    tok_k = rng.standard_normal((pairs, 1, 128)).astype(np.float16)
    tok_v = rng.standard_normal((pairs, 1, 128)).astype(np.float16)
    pk.packkv_append_token(cache, to_dev(tok_k), to_dev(tok_v))
    return cache, tok_v


def test_noalloc_capacity_limit(pk):
    """Find the largest number of (sequence, head) pairs that fits the fixed scratch with
    G = 8 (a refusal is decided on the host, before any launch); that call must give the
    right result and one more pair must be refused."""
    G = 8
    out_cache = {}

    def accepted(pairs):
        cache, tok_v = _tail_only_cache(pk, pairs, G, pairs)
        p = torch.ones((pairs, G, 4), device="cuda")
        out = torch.zeros((pairs, G, 128), device="cuda")
        try:
            pk.packkv_pv_gemv_noalloc(cache, p, out)
        except pk.PackKVError as err:
            assert err.status == pk.ERR_CAPACITY
            return False
        torch.cuda.synchronize()
        out_cache[pairs] = (out.cpu().numpy(), tok_v)
        return True

    lo, hi = 1, 1 << 13          # 8192 pairs need (>= 8192) * 8 * 512 B > 8 MiB
    assert accepted(lo) and not accepted(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if accepted(mid):
            lo = mid
        else:
            hi = mid
    # need = (warps + pairs) * G * 512 <= 8 MiB with warps >= 1: at most 2047 pairs
    assert 1 <= lo <= (8 << 20) // (G * 512) - 1
    out, tok_v = out_cache[lo]
    # p = 1 on the single token: out = that token's V value in fp32, for every head
    want = np.broadcast_to(tok_v.astype(np.float64), (lo, 1, 128))
    assert np.array_equal(out, np.broadcast_to(want, (lo, G, 128)).astype(np.float32))
    with pytest.raises(pk.PackKVError) as err:
        cache, _ = _tail_only_cache(pk, lo + 1, G, 0)
        pk.packkv_pv_gemv_noalloc(cache, torch.ones((lo + 1, G, 4), device="cuda"),
                                  torch.zeros((lo + 1, G, 128), device="cuda"))
    assert err.value.status == pk.ERR_CAPACITY


_FRESH = r'''
import sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import oracle as O
from decode_gemv_packkv_b200 import synth
from decode_gemv_packkv_b200 import packkv as pk
from parity_util import assert_within_terms
# the cache's records come from the oracle, copied in with torch: the library's first
# device call in this process is packkv_pv_gemv_noalloc
B, H, G, bits = 1, 2, 2, 4
k, v, _ = synth.small_case(4242, B, H, G, 3 * 128 + 20, structured=True)
oc = O.OracleCache(B, H, 4, bits)
oc.encode_blocks(k[:, :, :384], v[:, :, :384], 3)
for t in range(384, k.shape[2]):
    oc.append_token(k[:, :, t], v[:, :, t])
cache = pk.PackKVCache(B, H, 4, bits, arena_bytes=len(oc.v_arena))
cache.v_arena.copy_(torch.frombuffer(bytearray(oc.v_arena), dtype=torch.uint8))
cache.v_index.copy_(torch.from_numpy(oc.v_index.view(np.int32)))
cache.v_tail.copy_(torch.from_numpy(oc.v_tail))
cache.s.n_blocks, cache.s.tail_len = oc.n_blocks, oc.tail_len
T = oc.tokens
p = np.random.default_rng(1).random((B, H * G, T)).astype(np.float32)
pd = torch.zeros((B, H * G, (T + 3) // 4 * 4), device="cuda")
pd[:, :, :T] = torch.from_numpy(p).cuda()
for call in range(2):
    out = torch.full((B, H * G, 128), 3.0, device="cuda")
    pk.packkv_pv_gemv_noalloc(cache, pd, out)
    want, terms = O.cache_pv(oc, p)
    assert_within_terms(out.cpu().numpy(), want, terms, "first calls in a fresh process")
print("FRESH_OK")
'''


def test_noalloc_first_call_in_a_fresh_process(pk):
    code = "ROOT = " + repr(ROOT) + "\n" + _FRESH
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0 and "FRESH_OK" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]
