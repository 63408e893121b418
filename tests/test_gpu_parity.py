"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Encoder: records, index, arena ends and permutations bit-exact.  GEMVs: every
element within 1e-3 * sum|terms| (packed-cache format v1, section 7).  Small cases span
several blocks, pack groups and a ragged tail; the full workload sizes are
checked in the launch configuration the benchmark times, on sampled blocks the
oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle as O
from decode_gemv_packkv_b200 import synth
from parity_util import assert_within_terms, compare_encoder, gpu_record, gpu_records, to_dev

pytestmark = pytest.mark.gpu

SCALE = 1.0 / np.sqrt(128.0)


@pytest.fixture(scope="module")
def pk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import packkv
    return packkv


def _build(pk, k, v, bits, key=O.KEY_K_SUM, max_blocks=None, keep_perm=True, arena_bytes=None,
           unit_mode=O.UNITS_FOR):
    B, H, T, _ = k.shape
    nb_total = T // 128
    mb = max_blocks or max(1, nb_total + 1)
    cache = pk.PackKVCache(B, H, mb, bits, reorder_key=key, keep_perm=keep_perm, arena_bytes=arena_bytes,
                           unit_mode=unit_mode)
    pk.prefill(cache, to_dev(k), to_dev(v))
    ocache = O.OracleCache(B, H, mb, bits, key, unit_mode=unit_mode)
    ocache.encode_blocks(k[:, :, :nb_total * 128], v[:, :, :nb_total * 128], nb_total)
    for t in range(nb_total * 128, T):
        ocache.append_token(k[:, :, t], v[:, :, t])
    return cache, ocache


def _qk(pk, cache, q, ld=None):
    B, Hq, _ = q.shape
    ld = ld or ((cache.tokens + 3) // 4 * 4)
    scores = torch.full((B, Hq, ld), 7.0, dtype=torch.float32, device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    torch.cuda.synchronize()
    return scores.cpu().numpy()


def _pv(pk, cache, p):
    B, Hq, T = p.shape
    ld = (T + 3) // 4 * 4
    pd = torch.zeros((B, Hq, ld), dtype=torch.float32, device="cuda")
    pd[:, :, :T] = to_dev(p.astype(np.float32))
    out = torch.full((B, Hq, 128), 7.0, dtype=torch.float32, device="cuda")
    pk.packkv_pv_gemv(cache, pd, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


# ----------------------------------------------------------------------------- encoder
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("structured", [False, True])
@pytest.mark.parametrize("key", [O.KEY_IDENTITY, O.KEY_K_SUM, O.KEY_KV_SUM])
def test_encoder_bit_exact(pk, bits, structured, key):
    k, v, _ = synth.small_case(100 + bits + 3 * key, 2, 3, 1, 512, structured=structured)
    cache, ocache = _build(pk, k, v, bits, key)
    compare_encoder(cache, ocache)
    assert pk.packkv_get_status(cache) == 0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_width_only_units(pk, bits):
    """The width-only unit mode (base 0, width of the largest code): records bit-exact
    with the oracle, and the products over them (every decode path reads them as the
    v1 units they are) within 1e-3 * sum|terms|."""
    k, v, q = synth.small_case(150 + bits, 3, 4, 2, 5 * 128 + 21, structured=True)
    cache, ocache = _build(pk, k, v, bits, unit_mode=O.UNITS_WIDTH_ONLY)
    compare_encoder(cache, ocache)
    got = _qk(pk, cache, q)
    ref, terms = O.cache_qk(ocache, q, SCALE)
    T = ocache.tokens
    assert_within_terms(got[:, :, :T], ref, terms, "scores, width-only units")
    p = O.softmax(ref)
    ref_o, terms_o = O.cache_pv(ocache, p)
    assert_within_terms(_pv(pk, cache, p), ref_o, terms_o, "p·V, width-only units")
    att = torch.zeros((3, 8, 128), device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, att)
    ref_a, terms_a = O.cache_attention(ocache, q, SCALE)
    assert_within_terms(att.cpu().numpy(), ref_a, terms_a, "attention, width-only units")
    assert pk.packkv_get_status(cache) == 0


def test_encoder_two_calls_append_after_arena_end(pk):
    """A second encode call appends after the first call's records (arena order)."""
    k, v, _ = synth.small_case(5, 2, 2, 1, 768, structured=True)
    cache = pk.PackKVCache(2, 2, 8, 3, keep_perm=True)
    ocache = O.OracleCache(2, 2, 8, 3)
    for lo, n in ((0, 2), (256, 3), (640, 1)):
        sl = slice(lo, lo + 128 * n)
        pk.packkv_encode_block(cache, to_dev(k[:, :, sl].copy()), to_dev(v[:, :, sl].copy()), n)
        ocache.encode_blocks(k[:, :, sl], v[:, :, sl], n)
    compare_encoder(cache, ocache)


# ----------------------------------------------------------------------------- q·Kᵀ
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("structured", [False, True])
def test_qk_parity(pk, bits, group, structured):
    tail = {1: 0, 2: 37, 4: 127, 8: 1}[group]
    k, v, q = synth.small_case(200 + bits * 10 + group, 2, 2, group, 3 * 128 + tail, structured=structured)
    cache, ocache = _build(pk, k, v, bits)
    got = _qk(pk, cache, q)
    ref, terms = O.cache_qk(ocache, q, SCALE)
    T = ocache.tokens
    assert_within_terms(got[:, :, :T], ref, terms, "scores")
    assert np.all(got[:, :, T:] == 7.0), "wrote past T"


def test_qk_leading_dimension_and_tail_only(pk):
    k, v, q = synth.small_case(9, 1, 2, 2, 77)
    cache, ocache = _build(pk, k, v, 4)
    assert cache.n_blocks == 0 and cache.tail_len == 77
    got = _qk(pk, cache, q, ld=200)
    ref, terms = O.cache_qk(ocache, q, SCALE)
    assert_within_terms(got[:, :, :77], ref, terms, "tail scores")
    assert np.all(got[:, :, 77:] == 7.0)


# ----------------------------------------------------------------------------- p·V
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("structured", [False, True])
def test_pv_parity(pk, bits, group, structured):
    tail = {1: 5, 2: 0, 4: 64, 8: 127}[group]
    k, v, q = synth.small_case(300 + bits * 10 + group, 2, 2, group, 5 * 128 + tail, structured=structured)
    cache, ocache = _build(pk, k, v, bits)
    scores, _ = O.cache_qk(ocache, q, SCALE)
    p = O.softmax(scores).astype(np.float32)          # storage order, same fp32 p on both sides
    got = _pv(pk, cache, p)
    ref, terms = O.cache_pv(ocache, p)
    assert_within_terms(got, ref, terms, "p·V (softmax p)")
    rng = np.random.default_rng(bits + group)
    p2 = rng.standard_normal(p.shape).astype(np.float32)  # signed weights: cancellation
    got2 = _pv(pk, cache, p2)
    ref2, terms2 = O.cache_pv(ocache, p2)
    assert_within_terms(got2, ref2, terms2, "p·V (signed p)")


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pv_zero_and_tiny_weights(pk, bits):
    """Whole records with p = 0, records with p far below any useful magnitude
    (1e-35, under the digit-scale floor) and ordinary records side by side: the
    result stays finite and within the tolerance (the tiny terms are negligible)."""
    k, v, q = synth.small_case(40 + bits, 1, 2, 2, 4 * 128 + 9)
    cache, ocache = _build(pk, k, v, bits)
    rng = np.random.default_rng(bits)
    p = np.zeros((1, 4, cache.tokens), np.float32)
    p[..., 0:128] = rng.random((1, 4, 128)).astype(np.float32)      # block 0: ordinary
    p[..., 256:384] = np.float32(1e-35)                             # block 2: tiny
    p[..., 512:] = rng.random((1, 4, cache.tokens - 512)).astype(np.float32)  # the tail
    got = _pv(pk, cache, p)
    assert np.all(np.isfinite(got))
    ref, terms = O.cache_pv(ocache, p)
    assert_within_terms(got, ref, terms, "p·V (zero and tiny records)")
    assert pk.packkv_get_status(cache) == 0


def test_pv_is_deterministic_with_a_dirty_workspace(pk):
    k, v, q = synth.small_case(12, 2, 4, 2, 20 * 128 + 3)
    cache, _ = _build(pk, k, v, 4, keep_perm=False)
    p = np.random.default_rng(0).random((2, 8, cache.tokens)).astype(np.float32)
    a = _pv(pk, cache, p)
    cache.workspace(8).fill_(0xAB)     # garbage left by someone else: no initialisation needed
    b = _pv(pk, cache, p)
    assert np.array_equal(a, b)


def test_empty_cache(pk):
    cache = pk.PackKVCache(1, 2, 4, 3)
    out = torch.full((1, 2, 128), 5.0, device="cuda")
    pk.packkv_pv_gemv(cache, torch.zeros((1, 2, 4), device="cuda"), out)
    scores = torch.full((1, 2, 4), 5.0, device="cuda")
    pk.packkv_qk_gemv(cache, torch.zeros((1, 2, 128), dtype=torch.float16, device="cuda"), 1.0, scores)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(scores == 5.0)


# ----------------------------------------------------------------------------- growth
@pytest.mark.parametrize("bits", [2, 4])
def test_streaming_append_matches_oracle(pk, bits):
    """Token-by-token growth across block boundaries ([Abs]: dynamic growth)."""
    B, H, G = 2, 2, 2
    k, v, q = synth.small_case(41 + bits, B, H, G, 128 + 300, structured=(bits == 2))
    cache = pk.PackKVCache(B, H, 4, bits, keep_perm=True)
    ocache = O.OracleCache(B, H, 4, bits)
    pk.packkv_encode_block(cache, to_dev(k[:, :, :128].copy()), to_dev(v[:, :, :128].copy()), 1)
    ocache.encode_blocks(k[:, :, :128], v[:, :, :128], 1)
    kd, vd = to_dev(k), to_dev(v)
    for t in range(128, 428):
        pk.packkv_append_token(cache, kd[:, :, t].contiguous(), vd[:, :, t].contiguous())
        ocache.append_token(k[:, :, t], v[:, :, t])
        if t in (128, 254, 255, 256, 383, 384, 427):
            assert (cache.n_blocks, cache.tail_len) == (ocache.n_blocks, ocache.tail_len)
            got = _qk(pk, cache, q)
            ref, terms = O.cache_qk(ocache, q, SCALE)
            assert_within_terms(got[:, :, :ocache.tokens], ref, terms, f"scores at t={t}")
            p = O.softmax(ref).astype(np.float32)
            got_o = _pv(pk, cache, p)
            ref_o, terms_o = O.cache_pv(ocache, p)
            assert_within_terms(got_o, ref_o, terms_o, f"out at t={t}")
    compare_encoder(cache, ocache)
    with pytest.raises(pk.PackKVError):
        for t in range(428, 428 + 128):   # the 4th block would exceed max_blocks=4? 3 + 1 fits; a 5th does not
            pk.packkv_append_token(cache, kd[:, :, 0].contiguous(), vd[:, :, 0].contiguous())
        for t in range(128):
            pk.packkv_append_token(cache, kd[:, :, 0].contiguous(), vd[:, :, 0].contiguous())


# ----------------------------------------------------------------------------- device-detected errors
def test_arena_overflow_is_detected_on_device(pk):
    k, v, q = synth.small_case(77, 1, 2, 1, 256)
    cache = pk.PackKVCache(1, 2, 4, 4, arena_bytes=3 * 8720)   # room for 3 of the 4 records
    pk.packkv_encode_block(cache, to_dev(k), to_dev(v), 2)
    bits = pk.packkv_get_status(cache)
    assert bits & pk.DEV_CAPACITY
    assert cache.arena_used() == (0, 0)
    idx = cache.k_index.cpu().numpy().view(np.uint32)
    assert np.all(idx[0, :, :2, 0] == 0xFFFFFFFF)
    scores = torch.zeros((1, 2, 256), device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), 1.0, scores)
    assert torch.all(torch.isnan(scores))
    assert pk.packkv_get_status(cache) & pk.DEV_BAD_RECORD
    assert pk.packkv_get_status(cache) == 0     # read-and-clear


@pytest.mark.parametrize("where,value", [("k", np.inf), ("k", -np.inf), ("v", np.nan), ("k", np.nan),
                                         ("v", -np.inf)])
def test_nonfinite_input_sets_status(pk, where, value):
    """A NaN or an infinity anywhere in a block sets the sticky non-finite bit; a clean
    block after it does not."""
    k, v, _ = synth.small_case(78, 1, 1, 1, 256)
    (k if where == "k" else v)[0, 0, 5, 7] = value
    cache = pk.PackKVCache(1, 1, 3, 4)
    pk.packkv_encode_block(cache, to_dev(k[:, :, :128].copy()), to_dev(v[:, :, :128].copy()), 1)
    assert pk.packkv_get_status(cache) & pk.DEV_NONFINITE
    pk.packkv_encode_block(cache, to_dev(k[:, :, 128:].copy()), to_dev(v[:, :, 128:].copy()), 1)
    assert pk.packkv_get_status(cache) == 0


# ----------------------------------------------------------------------------- full workload sizes
def _upload(w, tokens, structured=False):
    """K, V on the device for a workload, generated one (b, h) slice at a time."""
    kd = torch.empty((w.batch, w.kv_heads, tokens, 128), dtype=torch.float16, device="cuda")
    vd = torch.empty_like(kd)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            ks, vs = synth.kv_slice(w.seed, w.kv_heads, b, h, tokens, structured=structured)
            kd[b, h].copy_(torch.from_numpy(ks))
            vd[b, h].copy_(torch.from_numpy(vs))
    return kd, vd


def _sampled_check(pk, w, bits, kd, vd, cache, samples, full_bh):
    """Encoder records, scores and outputs on sampled blocks (+ one whole sequence)."""
    q = synth.queries(w)
    G = w.group
    T = cache.tokens
    scores = torch.empty((w.batch, w.q_heads, T), dtype=torch.float32, device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    # p nonzero on the sampled blocks only: the oracle needs just those blocks
    p = np.zeros((w.batch, w.q_heads, T), np.float32)
    rng = np.random.default_rng(bits)
    for (b, h, i) in samples:
        p[b, h * G:(h + 1) * G, i * 128:(i + 1) * 128] = rng.random((G, 128), dtype=np.float32)
    out = torch.empty((w.batch, w.q_heads, 128), dtype=torch.float32, device="cuda")
    pk.packkv_pv_gemv(cache, to_dev(p), out)
    torch.cuda.synchronize()
    s_np = scores.cpu().numpy()
    o_np = out.cpu().numpy()
    karena, kindex = gpu_records(cache, "k")
    varena, vindex = gpu_records(cache, "v")
    o_ref = np.zeros_like(o_np, dtype=np.float64)
    o_terms = np.zeros_like(o_ref)
    for (b, h, i) in samples:
        kb = kd[b, h, i * 128:(i + 1) * 128].cpu().numpy()
        vb = vd[b, h, i * 128:(i + 1) * 128].cpu().numpy()
        k_rec, v_rec, _ = O.encode_block(kb, vb, bits)
        assert gpu_record(karena, kindex, b, h, i) == k_rec, f"K record {(b, h, i)}"
        assert gpu_record(varena, vindex, b, h, i) == v_rec, f"V record {(b, h, i)}"
        kdec = O.dequant_k(O.parse_record(k_rec))
        vdec = O.dequant_v(O.parse_record(v_rec))
        ref, terms = O.qk_scores(q[b, h * G:(h + 1) * G], kdec, SCALE)
        assert_within_terms(s_np[b, h * G:(h + 1) * G, i * 128:(i + 1) * 128], ref, terms, f"scores {(b, h, i)}")
        o, t = O.pv_out(p[b, h * G:(h + 1) * G, i * 128:(i + 1) * 128], vdec)
        o_ref[b, h * G:(h + 1) * G] += o
        o_terms[b, h * G:(h + 1) * G] += t
    assert_within_terms(o_np, o_ref, o_terms, "p·V on sampled blocks")
    # one whole sequence, dense softmax p
    b, h = full_bh
    ocache = O.OracleCache(1, 1, cache.n_blocks, bits)
    nbk = cache.n_blocks
    ocache.encode_blocks(kd[b:b + 1, h:h + 1, :nbk * 128].cpu().numpy(), vd[b:b + 1, h:h + 1, :nbk * 128].cpu().numpy(),
                         nbk)
    ref, terms = O.cache_qk(ocache, q[b:b + 1, h * G:(h + 1) * G], SCALE)
    assert_within_terms(s_np[b:b + 1, h * G:(h + 1) * G], ref, terms, "scores, whole sequence")
    pdense = np.zeros((w.batch, w.q_heads, T), np.float32)
    pdense[b, h * G:(h + 1) * G] = O.softmax(ref[0]).astype(np.float32)
    pk.packkv_pv_gemv(cache, to_dev(pdense), out)
    ref_o, terms_o = O.cache_pv(ocache, pdense[b:b + 1, h * G:(h + 1) * G])
    assert_within_terms(out.cpu().numpy()[b:b + 1, h * G:(h + 1) * G], ref_o, terms_o, "p·V, whole sequence")
    assert np.all(np.isfinite(s_np))
    assert pk.packkv_get_status(cache) == 0
    return ocache


@pytest.mark.parametrize("wid,bits", [(0, 4), (1, 4), (2, 4), (2, 2), (3, 3)])
def test_full_workload_sampled(pk, wid, bits):
    w = synth.WORKLOADS[wid]
    kd, vd = _upload(w, w.seq)
    nb = w.seq // 128
    cache = pk.PackKVCache(w.batch, w.kv_heads, nb, bits)
    pk.packkv_encode_block(cache, kd, vd, nb)
    rng = np.random.default_rng(wid)
    samples = {(int(rng.integers(w.batch)), int(rng.integers(w.kv_heads)), int(rng.integers(nb)))
               for _ in range(6)}
    samples |= {(0, 0, 0), (w.batch - 1, w.kv_heads - 1, nb - 1)}
    _sampled_check(pk, w, bits, kd, vd, cache, sorted(samples), (w.batch - 1, w.kv_heads // 2))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_streaming_workload(pk, bits):
    """Batch 4 x 32 heads, prefill 8192 then 4096 appended tokens; GEMVs every step,
    checked against the oracle at steps 0, 1, 127, 128, 129, every 512th and the last
    on two sequences, and every block encoded during decode checked bit-exact there."""
    w = synth.WORKLOADS[4]
    total = w.seq + w.decode_steps
    kd, vd = _upload(w, total)
    nb_max = total // 128
    cache = pk.PackKVCache(w.batch, w.kv_heads, nb_max, bits)
    pk.packkv_encode_block(cache, kd[:, :, :w.seq].contiguous(), vd[:, :, :w.seq].contiguous(), w.seq // 128)
    G = w.group
    check_steps = {0, 1, 127, 128, 129, w.decode_steps - 1} | set(range(0, w.decode_steps, 512))
    seqs = [(0, 3), (w.batch - 1, w.kv_heads - 1)]
    oc = {}
    for (b, h) in seqs:
        o = O.OracleCache(1, 1, nb_max, bits)
        o.encode_blocks(kd[b:b + 1, h:h + 1, :w.seq].cpu().numpy(), vd[b:b + 1, h:h + 1, :w.seq].cpu().numpy(),
                        w.seq // 128)
        oc[(b, h)] = o
    k_np = {bh: kd[bh[0], bh[1], w.seq:].cpu().numpy() for bh in seqs}
    v_np = {bh: vd[bh[0], bh[1], w.seq:].cpu().numpy() for bh in seqs}
    ld = (total + 3) // 4 * 4
    scores = torch.empty((w.batch, w.q_heads, ld), dtype=torch.float32, device="cuda")
    out = torch.empty((w.batch, w.q_heads, 128), dtype=torch.float32, device="cuda")
    for step in range(w.decode_steps):
        t = w.seq + step
        pk.packkv_append_token(cache, kd[:, :, t].contiguous(), vd[:, :, t].contiguous())
        for bh in seqs:
            oc[bh].append_token(k_np[bh][step][None, None], v_np[bh][step][None, None])
        q = synth.queries(w, step)
        pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
        T = cache.tokens
        p = torch.softmax(scores[:, :, :T], dim=-1)
        pfull = torch.zeros_like(scores)
        pfull[:, :, :T] = p
        pk.packkv_pv_gemv(cache, pfull, out)
        if step in check_steps:
            s_np = scores.cpu().numpy()
            p_np = pfull.cpu().numpy()
            o_np = out.cpu().numpy()
            for (b, h), o in oc.items():
                assert o.tokens == T
                ref, terms = O.cache_qk(o, q[b:b + 1, h * G:(h + 1) * G], SCALE)
                assert_within_terms(s_np[b:b + 1, h * G:(h + 1) * G, :T], ref, terms, f"scores step {step}")
                ref_o, terms_o = O.cache_pv(o, p_np[b:b + 1, h * G:(h + 1) * G, :T])
                assert_within_terms(o_np[b:b + 1, h * G:(h + 1) * G], ref_o, terms_o, f"out step {step}")
    karena, kindex = gpu_records(cache, "k")
    varena, vindex = gpu_records(cache, "v")
    for (b, h), o in oc.items():
        for i in range(w.seq // 128, o.n_blocks):
            assert gpu_record(karena, kindex, b, h, i) == o.record("k", 0, 0, i)
            assert gpu_record(varena, vindex, b, h, i) == o.record("v", 0, 0, i)
    assert pk.packkv_get_status(cache) == 0


# ----------------------------------------------------------------------------- compressed records at scale
@pytest.mark.parametrize("bits", [4, 2])
def test_full_size_structured_cache(pk, bits):
    """The 32-head 32k-token shape on run-structured inputs, where most records are
    compressed (unit widths 0..b) and some raw, so warps run compressed and raw records
    back to back in the launch configuration the benchmark uses: records on sampled
    blocks bit-exact, q·Kᵀ and p·V on sampled blocks and one whole sequence, and the
    fused attention over that sequence."""
    w = synth.WORKLOADS[1]
    kd, vd = _upload(w, w.seq, structured=True)
    nb = w.seq // 128
    cache = pk.PackKVCache(w.batch, w.kv_heads, nb, bits)
    pk.packkv_encode_block(cache, kd, vd, nb)
    raw = O.raw_record_bytes(bits) // 16
    for which in ("k", "v"):
        lens = gpu_records(cache, which)[1][..., 1]
        assert np.any(lens < raw), f"{which}: no compressed record"
    assert np.any(gpu_records(cache, "k")[1][..., 1] == raw), "K: no raw record"
    rng = np.random.default_rng(100 + bits)
    samples = {(0, int(rng.integers(w.kv_heads)), int(rng.integers(nb))) for _ in range(6)}
    samples |= {(0, 0, 0), (0, w.kv_heads - 1, nb - 1)}
    h = 7
    oc = _sampled_check(pk, w, bits, kd, vd, cache, sorted(samples), (0, h))
    q = synth.queries(w)
    out = torch.zeros((w.batch, w.q_heads, 128), device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, out)
    ref, terms = O.cache_attention(oc, q[0:1, h:h + 1], SCALE)
    assert_within_terms(out.cpu().numpy()[0:1, h:h + 1], ref, terms, "attention, whole structured sequence")
    assert pk.packkv_get_status(cache) == 0


@pytest.mark.parametrize("bits,group", [(4, 1), (2, 4), (3, 2)])
def test_many_items_per_warp(pk, bits, group):
    """2048 (sequence, head) pairs of 64 blocks plus a 57-token tail: 133k items, about
    45 per warp, so every warp crosses many (sequence, head) boundaries, reloads its
    window of index entries and runs compressed records, raw records and tails in one
    pass.  Eight distinct structured sequences are tiled over the pairs (the oracle
    decodes each once); scores, outputs and the fused attention are checked on a
    contiguous run of pairs and on scattered ones."""
    B, H, nb, tail, n_distinct = 64, 32, 64, 57, 8
    T = nb * 128 + tail
    G = group
    ks, vs = [], []
    for i in range(n_distinct):
        k1, v1 = synth.kv_slice(7000 + 10 * bits + G, n_distinct, 0, i, T, structured=True)
        ks.append(torch.from_numpy(k1))
        vs.append(torch.from_numpy(v1))
    kd = torch.empty((B, H, T, 128), dtype=torch.float16, device="cuda")
    vd = torch.empty_like(kd)
    for p_ in range(B * H):
        kd.view(B * H, T, 128)[p_].copy_(ks[p_ % n_distinct], non_blocking=True)
        vd.view(B * H, T, 128)[p_].copy_(vs[p_ % n_distinct], non_blocking=True)
    cache = pk.PackKVCache(B, H, nb + 1, bits)
    pk.packkv_encode_block(cache, kd[:, :, :nb * 128].contiguous(), vd[:, :, :nb * 128].contiguous(), nb)
    for t in range(nb * 128, T):
        pk.packkv_append_token(cache, kd[:, :, t].contiguous(), vd[:, :, t].contiguous())
    del kd, vd
    oc = []
    for i in range(n_distinct):
        o = O.OracleCache(1, 1, nb + 1, bits)
        o.encode_blocks(ks[i][:nb * 128].numpy()[None, None], vs[i][:nb * 128].numpy()[None, None], nb)
        for t in range(nb * 128, T):
            o.append_token(ks[i][t].numpy()[None, None], vs[i][t].numpy()[None, None])
        oc.append(o)
    rng = np.random.default_rng(bits * 10 + G)
    q = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    ld = (T + 3) // 4 * 4
    scores = torch.empty((B, H * G, ld), device="cuda")
    pk.packkv_qk_gemv(cache, to_dev(q), SCALE, scores)
    p = rng.random((B, H * G, ld)).astype(np.float32)
    p[:, :, T:] = 0
    out = torch.empty((B, H * G, 128), device="cuda")
    pk.packkv_pv_gemv(cache, to_dev(p), out)
    att = torch.empty((B, H * G, 128), device="cuda")
    pk.packkv_attention_decode(cache, to_dev(q), SCALE, att)
    s_np, o_np, a_np = scores.cpu().numpy(), out.cpu().numpy(), att.cpu().numpy()
    pairs = list(range(600, 760)) + [int(x) for x in rng.integers(0, B * H, 40)] + [0, B * H - 1]
    for pr in sorted(set(pairs)):
        b, h = divmod(pr, H)
        o = oc[pr % n_distinct]
        hs = slice(h * G, (h + 1) * G)
        ref, terms = O.cache_qk(o, q[b:b + 1, hs], SCALE)
        assert_within_terms(s_np[b:b + 1, hs, :T], ref, terms, f"scores of pair {pr}")
        ref, terms = O.cache_pv(o, p[b:b + 1, hs, :T])
        assert_within_terms(o_np[b:b + 1, hs], ref, terms, f"p·V of pair {pr}")
        ref, terms = O.cache_attention(o, q[b:b + 1, hs], SCALE)
        assert_within_terms(a_np[b:b + 1, hs], ref, terms, f"attention of pair {pr}")
    assert pk.packkv_get_status(cache) == 0
