"""Benchmark of the PackKV decode path on B200: fused unpack + GEMV throughput.

One step = packkv_qk_gemv then packkv_pv_gemv over the whole packed cache of
the workload (every sequence and head), i.e. the two decode-time products of
the PackKV pages (Figure 1 attention, Figure 2 fused decompression + GEMV).
Headline workload: Llama-7B-style decode layer, 32 MHA heads, head_dim 128,
batch 1, 32768 cached tokens, 4-bit codes (synthetic K/V with the per-channel
outlier distribution; see decode_gemv_packkv_b200/synth.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ID] [--bits B] [--no-sub] [--no-cpu-baseline]

Prints one JSON line (rank 0).  Timing: W untimed steps, then K steps bracketed
by a barrier and a device synchronize, CUDA events on the launching stream,
max over ranks.  Inputs exceed L2: steps rotate over several cache copies.
The line also carries one sub-record per other workload ("workloads": the
single-head, GQA 4/2-bit, batched 3-bit and streaming-growth shapes, plus the
headline shape on run-structured inputs, where most records are compressed),
each timed per kernel the same way.  --impl reference times the CPU oracle on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_gemv_packkv_b200 import synth  # noqa: E402

METRIC = "fused unpack+GEMV tokens/s (q·Kᵀ + p·V over the packed KV cache)"
UNIT = "tokens/s"
SCALE = 1.0 / float(np.sqrt(128.0))
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own independent batch (weak scaling, no data-path collective)."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: the tokens every rank decoded in one step over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# kernels of this library launched by one step: q·Kᵀ (1), p·V (2: the split pass and its reduce)
KERNELS_PER_STEP = 3

# wall-clock budget of the reference arm (warm-up + timed steps), seconds
REFERENCE_SECONDS = 150.0


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks
def physical_gpu_index(local_index: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if local_index < len(ids) and ids[local_index].isdigit():
        return int(ids[local_index])
    return local_index


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu_index = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [[c.strip() for c in line.split(",")] for line in out.strip().splitlines() if line.strip()]
        sm = [float(r[0]) for r in rows if r and r[0].replace(".", "", 1).isdigit()]
        mx = [float(r[1]) for r in rows if len(r) > 1 and r[1].replace(".", "", 1).isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 4 + i and r[4 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ measured peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return 6650.0, "fallback 6.65 TB/s"


# DRAM bytes (read + write) per launch of pv_kernel, the first pass of packkv_pv_gemv,
# measured by ncu on this build's kernels (dram__bytes_read.sum + dram__bytes_write.sum,
# mean of two launches on the 32-head 32k-token 4-bit cache; summary in
# profiles/launches__bench_mha32_seq32k_b4.md).  The q·Kᵀ entry serves when q·Kᵀ is the
# dominant kernel.  None for
# other workloads, and None whenever the kernel has changed since the capture.
DRAM_TRAFFIC = {
    ("llama7b-decode mha b1 h32 d128 seq32768 4-bit", 4, "pv"): 75_790_848,
    ("llama7b-decode mha b1 h32 d128 seq32768 4-bit", 4, "qk"): 72_169_088,
}


# ------------------------------------------------------------------ the CUDA path: helpers
def upload(w, tokens, dev, structured=False):
    """K, V [B, Hkv, tokens, 128] fp16 on the device, generated one (b, h) slice at a time."""
    import torch
    kd = torch.empty((w.batch, w.kv_heads, tokens, 128), dtype=torch.float16, device=dev)
    vd = torch.empty_like(kd)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            ks, vs = synth.kv_slice(w.seed, w.kv_heads, b, h, tokens, structured=structured)
            kd[b, h].copy_(torch.from_numpy(ks))
            vd[b, h].copy_(torch.from_numpy(vs))
    return kd, vd


def copies_for(bytes_per_launch: int, cap: int = 2048) -> int:
    """Cache copies to rotate so that a launch never finds its records in L2: together
    at least 2.5x the 126 MB L2 between two reads of the same bytes."""
    return int(min(cap, max(1, int(np.ceil(2.5 * L2_BYTES / max(1, bytes_per_launch))))))


def timed_ms(dev, fn, pre_sleep=True) -> float:
    """CUDA-event time of fn() on the current stream; a short device sleep first keeps
    the stream busy while the host enqueues (graph upload stays off the clock)."""
    import torch
    cur = torch.cuda.current_stream(dev)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pre_sleep:
        torch.cuda._sleep(20_000_000)
    a.record(cur)
    fn()
    b_.record(cur)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b_)


def median_ms(dev, fn, reps: int = 5) -> float:
    """Median of `reps` CUDA-event timings of fn() (per-kernel sub-record times)."""
    return statistics.median(timed_ms(dev, fn) for _ in range(reps))


def capture(dev, fn):
    """A CUDA graph of fn() (run once eagerly on a side stream first)."""
    import torch
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


class CacheSet:
    """R copies of one workload's packed cache with their own q, p, scores, out and
    workspaces, for rotation (every launch reads HBM)."""

    def __init__(self, pk, dev, w, bits, kd, vd, R, key=None, p_np=None):
        import torch
        self.pk, self.dev, self.w, self.bits = pk, dev, w, bits
        B, Hq, Hkv, T = w.batch, w.q_heads, w.kv_heads, kd.shape[2]
        self.B, self.Hq, self.Hkv, self.T = B, Hq, Hkv, T
        nb = T // 128
        key = pk.KEY_K_SUM if key is None else key
        probe = pk.PackKVCache(B, Hkv, nb, bits, reorder_key=key)
        pk.packkv_encode_block(probe, kd, vd, nb)
        self.k_used, self.v_used = probe.arena_used()
        self.k_lens = probe.k_index[..., 1].cpu().numpy().astype(np.int64)
        self.v_lens = probe.v_index[..., 1].cpu().numpy().astype(np.int64)
        del probe
        self.caches = []
        for _ in range(R):
            c = pk.PackKVCache(B, Hkv, nb, bits, reorder_key=key, arena_bytes=max(self.k_used, self.v_used) + 16)
            pk.packkv_encode_block(c, kd, vd, nb)
            self.caches.append(c)
        assert all(pk.packkv_get_status(c) == 0 for c in self.caches)
        self.R = R
        self.ld = (T + 3) // 4 * 4
        self.q = [torch.from_numpy(synth.queries(w, i)).to(dev) for i in range(R)]
        if p_np is None:
            p_np = synth.timing_probs(w, T)
        self.p = []
        for _ in range(R):
            t_ = torch.zeros((B, Hq, self.ld), dtype=torch.float32, device=dev)
            t_[:, :, :T] = torch.from_numpy(p_np).to(dev)
            self.p.append(t_)
        self.scores = [torch.empty((B, Hq, self.ld), dtype=torch.float32, device=dev) for _ in range(R)]
        self.outs = [torch.empty((B, Hq, 128), dtype=torch.float32, device=dev) for _ in range(R)]
        # one workspace serves every copy: the launches run one after another on one stream
        self.ws = [self.caches[0].workspace(Hq)] * R
        self.wsa = [self.caches[0].attention_workspace(Hq)] * R
        self.index_bytes = B * Hkv * nb * 8
        self.fp16_bytes = B * Hkv * T * 128 * 2

    def qk(self, i):
        self.pk.packkv_qk_gemv(self.caches[i], self.q[i], SCALE, self.scores[i])

    def pv(self, i):
        self.pk.packkv_pv_gemv(self.caches[i], self.p[i], self.outs[i], self.ws[i])

    def attn(self, i):
        self.pk.packkv_attention_decode(self.caches[i], self.q[i], SCALE, self.outs[i], self.wsa[i])

    def graph(self, *kinds, n=None):
        n = self.R if n is None else n

        def body():
            for i in range(n):
                for kd in kinds:
                    getattr(self, kd)(i)
        return capture(self.dev, body)

    def per_launch_ms(self, kind, min_launches=60):
        """Average time of one launch of `kind` over whole rotations of the copies (the
        median of five such timings)."""
        g = self.graph(kind)
        g.replay()
        reps = max(1, int(np.ceil(min_launches / self.R)))

        def run():
            for _ in range(reps):
                g.replay()
        return median_ms(self.dev, run) / (reps * self.R)

    def bytes(self):
        B, Hq, T = self.B, self.Hq, self.T
        qk_alg = self.k_used + self.index_bytes + B * Hq * 128 * 2 + B * Hq * T * 4
        pv_alg = self.v_used + self.index_bytes + B * Hq * T * 4 + B * Hq * 128 * 4
        attn_alg = self.k_used + self.v_used + 2 * self.index_bytes + B * Hq * 128 * 2 + B * Hq * 128 * 4
        return qk_alg, pv_alg, attn_alg


def cublas_ms(dev, kd, vd, G, reps=30):
    """Same-run cuBLAS fp16 GEMVs on the uncompressed cache (torch.matmul, fp32 accumulate):
    q·Kᵀ as [B*Hkv, T, 128] x [B*Hkv, 128, G] and p·V as [B*Hkv, G, T] x [B*Hkv, T, 128]."""
    import torch
    B, Hkv, T, _ = kd.shape
    kf = kd.view(B * Hkv, T, 128)
    vf = vd.view(B * Hkv, T, 128)
    qh = torch.randn((B * Hkv, 128, G), dtype=torch.float16, device=dev)
    ph = torch.rand((B * Hkv, G, T), dtype=torch.float16, device=dev)
    flush = torch.empty(3 * L2_BYTES // 4, dtype=torch.float32, device=dev) if 2 * kd.numel() < 3 * L2_BYTES else None
    for _ in range(3):
        torch.matmul(kf, qh)
        torch.matmul(ph, vf)
    torch.cuda.synchronize(dev)

    def one(fn):
        tot = 0.0
        for _ in range(reps):
            if flush is not None:
                flush.zero_()
            tot += timed_ms(dev, fn, pre_sleep=False)
        return tot / reps
    return one(lambda: torch.matmul(kf, qh)), one(lambda: torch.matmul(ph, vf))


def gemv_entry(ms, comp_bytes, alg_bytes, fp16_bytes, tokens, peak):
    return {"ms": ms, "tokens_per_s": tokens / (ms * 1e-3),
            "compressed_bytes": comp_bytes, "compressed_gbs": comp_bytes / (ms * 1e-3) / 1e9,
            "frac_hbm_compressed": comp_bytes / (ms * 1e-3) / 1e9 / peak,
            "algorithmic_bytes": alg_bytes, "algorithmic_gbs": alg_bytes / (ms * 1e-3) / 1e9,
            "frac_hbm_algorithmic": alg_bytes / (ms * 1e-3) / 1e9 / peak,
            "uncompressed_equiv_gbs": fp16_bytes / (ms * 1e-3) / 1e9}


def compression_entry(cs, bits):
    raw16 = (528 + 2048 * bits) // 16
    plain = 128 * 128 * 2 / (128 * 128 * bits / 8 + 512)
    cr_k = cs.fp16_bytes / (cs.k_used + cs.index_bytes)
    cr_v = cs.fp16_bytes / (cs.v_used + cs.index_bytes)
    return {"cr_k": cr_k, "cr_v": cr_v, "plain_quant_cr": plain, "vs_plain_quant_k": cr_k / plain - 1,
            "vs_plain_quant_v": cr_v / plain - 1, "raw_share_k": float(np.mean(cs.k_lens == raw16)),
            "raw_share_v": float(np.mean(cs.v_lens == raw16)),
            "k_record_bytes": int(cs.k_used), "v_record_bytes": int(cs.v_used)}


def workload_record(pk, dev, wid, bits, peak, structured=False, kd=None, vd=None, attention=True, w_override=None):
    """Per-kernel figures of one workload: q·Kᵀ, p·V and the fused attention, each
    timed alone over whole rotations of enough cache copies; compression; cuBLAS."""
    w = synth.WORKLOADS[wid] if w_override is None else w_override
    if kd is None:
        kd, vd = upload(w, w.seq, dev, structured)
    probe_bytes = w.batch * w.kv_heads * (w.seq // 128) * (528 + 2048 * bits)
    cs = CacheSet(pk, dev, w, bits, kd, vd, R=1)
    R = copies_for(min(cs.k_used, cs.v_used) or probe_bytes)
    if R > 1:
        cs = CacheSet(pk, dev, w, bits, kd, vd, R=R)
    B, T, G = w.batch, w.seq, w.group
    qk_ms = cs.per_launch_ms("qk")
    pv_ms = cs.per_launch_ms("pv")
    attn_ms = cs.per_launch_ms("attn") if attention else None
    qk_alg, pv_alg, attn_alg = cs.bytes()
    cb_qk, cb_pv = cublas_ms(dev, kd, vd, G)
    rec = {"workload": w.name, "bits": bits,
           "inputs": "run-structured (few levels per channel held for random runs)" if structured
           else "i.i.d. (the workload's distributions)",
           "batch": B, "q_heads": w.q_heads, "kv_heads": w.kv_heads, "seq": T, "copies": R,
           "qk": gemv_entry(qk_ms, cs.k_used + cs.index_bytes, qk_alg, cs.fp16_bytes, B * T, peak),
           "pv": gemv_entry(pv_ms, cs.v_used + cs.index_bytes, pv_alg, cs.fp16_bytes, B * T, peak),
           "step_tokens_per_s": B * T / ((qk_ms + pv_ms) * 1e-3),
           "compression": compression_entry(cs, bits),
           "cublas_fp16": {"qk_ms": cb_qk, "pv_ms": cb_pv, "qk_speedup": cb_qk / qk_ms, "pv_speedup": cb_pv / pv_ms}}
    if attention:
        rec["attention"] = {"ms": attn_ms, "tokens_per_s": B * T / (attn_ms * 1e-3),
                            "algorithmic_gbs": attn_alg / (attn_ms * 1e-3) / 1e9,
                            "frac_hbm_algorithmic": attn_alg / (attn_ms * 1e-3) / 1e9 / peak}
    del cs
    return rec


def streaming_record(pk, dev, bits, layers=3):
    """Streaming growth (batch 4 x 32 heads, prefill 8192 then 4096 decode steps): per
    decode step of one layer, packkv_append_token (which encodes the tail into a block
    every 128th step) then packkv_qk_gemv and packkv_pv_gemv over the blocks and the tail.
    `layers` independent caches step in turn, as the layers of a model do, so that a
    step does not find the previous step's records in L2.  All 4096 x layers steps are
    one CUDA graph, replayed once after an identical warm-up graph on other caches."""
    import torch
    w = synth.WORKLOADS[4]
    B, H, T0, S = w.batch, w.kv_heads, w.seq, w.decode_steps
    total = T0 + S
    kd, vd = upload(w, total, dev)
    nb0, nb_max = T0 // 128, total // 128
    ld = (total + 3) // 4 * 4
    q = torch.from_numpy(synth.queries(w, 0)).to(dev)
    p = torch.zeros((B, w.q_heads, ld), dtype=torch.float32, device=dev)
    p[:, :, :total] = torch.from_numpy(synth.timing_probs(w, total)).to(dev)
    scores = torch.empty((B, w.q_heads, ld), dtype=torch.float32, device=dev)
    out = torch.empty((B, w.q_heads, 128), dtype=torch.float32, device=dev)
    tok_k = [kd[:, :, t].contiguous() for t in range(T0, total)]
    tok_v = [vd[:, :, t].contiguous() for t in range(T0, total)]
    kpre, vpre = kd[:, :, :T0].contiguous(), vd[:, :, :T0].contiguous()

    def make_set():
        cs = []
        for _ in range(layers):
            c = pk.PackKVCache(B, H, nb_max, bits)
            pk.packkv_encode_block(c, kpre, vpre, nb0)
            c.workspace(w.q_heads)
            cs.append(c)
        return cs

    def steps(cs):
        for s in range(S):
            for c in cs:
                pk.packkv_append_token(c, tok_k[s], tok_v[s])
                pk.packkv_qk_gemv(c, q, SCALE, scores)
                pk.packkv_pv_gemv(c, p, out)

    graphs = []
    for _ in range(2):
        cs = make_set()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        s_ = torch.cuda.Stream(dev)
        s_.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.graph(g, stream=s_):
            steps(cs)
        torch.cuda.synchronize(dev)
        graphs.append((g, cs))
    graphs[0][0].replay()                 # warm-up on the first set
    torch.cuda.synchronize(dev)
    ms = timed_ms(dev, graphs[1][0].replay)
    cs = graphs[1][1]
    status = [pk.packkv_get_status(c) for c in cs]
    assert all(x == 0 for x in status), status
    assert all(c.n_blocks == nb_max and c.tail_len == 0 for c in cs)
    per_step = ms / (S * layers)
    # the encode a block boundary adds: one block per (sequence, head), timed alone
    enc = pk.PackKVCache(B, H, 2, bits)
    blk_k, blk_v = kd[:, :, :128].contiguous(), vd[:, :, :128].contiguous()

    def one_encode():
        pk.packkv_cache_reset(enc)
        pk.packkv_encode_block(enc, blk_k, blk_v, 1)
    for _ in range(3):
        one_encode()
    enc_ms = timed_ms(dev, lambda: [one_encode() for _ in range(50)]) / 50
    k_used = [c.arena_used()[0] for c in cs][0]
    del graphs, cs
    cb_qk, cb_pv = cublas_ms(dev, kd, vd, w.group)
    return {"workload": w.name, "bits": bits, "inputs": "i.i.d. (the workload's distributions)",
            "batch": B, "q_heads": w.q_heads, "kv_heads": H, "prefill": T0, "decode_steps": S, "layers": layers,
            "per_step_ms": per_step, "per_step_us": per_step * 1e3,
            "tokens_per_s": B / (per_step * 1e-3),
            "step": "packkv_append_token (+ the block encode every 128th step) + packkv_qk_gemv + packkv_pv_gemv "
                    "over blocks and tail, one layer; softmax between the products is the caller's and not included",
            "encode_one_block_per_pair_ms": enc_ms,
            "final_k_record_bytes": int(k_used),
            "cublas_fp16_at_final_length": {"qk_ms": cb_qk, "pv_ms": cb_pv, "sum_ms": cb_qk + cb_pv},
            "timing": f"one CUDA graph of {S} steps x {layers} layers (caches stepping in turn), "
                      "CUDA events, after a warm-up replay of an identical graph"}


def ragged_record(pk, dev, peak, bits=3):
    """Ragged batched decode: the batched shape (16 sequences x 32 heads, 3-bit) with
    each sequence's own length, a seeded multiple of 128 in [4096, 16384].  The cache
    is prefilled to 16384 tokens and each sequence's host counters are then set to
    its length (the records past it are not read).  q·Kᵀ, p·V and the fused attention
    are timed per launch; tokens/s counts every sequence's own tokens."""
    import torch
    w = synth.WORKLOADS[3]
    B, H, T = w.batch, w.kv_heads, w.seq
    nb = T // 128
    kd, vd = upload(w, T, dev)
    lens_blocks = np.random.default_rng(w.seed + 5).integers(32, nb + 1, B)
    probe = pk.PackKVCache(B, H, nb, bits, ragged=True)
    pk.packkv_encode_block(probe, kd, vd, nb)
    k_lens = probe.k_index[..., 1].cpu().numpy().astype(np.int64)
    v_lens = probe.v_index[..., 1].cpu().numpy().astype(np.int64)
    used_k = sum(int(k_lens[b, :, :lens_blocks[b]].sum()) * 16 for b in range(B))
    used_v = sum(int(v_lens[b, :, :lens_blocks[b]].sum()) * 16 for b in range(B))
    del probe
    R = copies_for(used_k)
    caches = []
    for _ in range(R):
        c = pk.PackKVCache(B, H, nb, bits, ragged=True)
        pk.packkv_encode_block(c, kd, vd, nb)
        for b in range(B):
            c._seq_blocks[b] = int(lens_blocks[b])
        caches.append(c)
    assert all(pk.packkv_get_status(c) == 0 for c in caches)
    del kd, vd
    Hq = w.q_heads
    ld = T
    q = [torch.from_numpy(synth.queries(w, i)).to(dev) for i in range(R)]
    p = torch.from_numpy(synth.timing_probs(w, T)).to(dev)
    scores = torch.empty((B, Hq, ld), dtype=torch.float32, device=dev)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
    ws, wsa = caches[0].workspace(Hq), caches[0].attention_workspace(Hq)

    def per_launch(fn):
        g = capture(dev, lambda: [fn(i) for i in range(R)])
        g.replay()
        reps = max(1, int(np.ceil(60 / R)))
        return median_ms(dev, lambda: [g.replay() for _ in range(reps)]) / (reps * R)
    qk_ms = per_launch(lambda i: pk.packkv_qk_gemv(caches[i], q[i], SCALE, scores))
    pv_ms = per_launch(lambda i: pk.packkv_pv_gemv(caches[i], p, out, ws))
    at_ms = per_launch(lambda i: pk.packkv_attention_decode(caches[i], q[i], SCALE, out, wsa))
    tokens = int(lens_blocks.sum()) * 128
    index_bytes = int(lens_blocks.sum()) * H * 8
    fp16 = tokens * H * 128 * 2
    qk_alg = used_k + index_bytes + B * Hq * 256 + int(lens_blocks.sum()) * 128 * Hq * 4
    pv_alg = used_v + index_bytes + int(lens_blocks.sum()) * 128 * Hq * 4 + B * Hq * 512
    del caches
    return {"workload": "ragged batched b16 h32 d128 seq 4096..16384 per sequence 3-bit", "bits": bits,
            "inputs": "i.i.d. (the workload's distributions)", "batch": B, "q_heads": Hq, "kv_heads": H,
            "tokens": tokens, "seq_lengths": [int(x) * 128 for x in lens_blocks], "copies": R,
            "qk": gemv_entry(qk_ms, used_k + index_bytes, qk_alg, fp16, tokens, peak),
            "pv": gemv_entry(pv_ms, used_v + index_bytes, pv_alg, fp16, tokens, peak),
            "attention": {"ms": at_ms, "tokens_per_s": tokens / (at_ms * 1e-3)},
            "step_tokens_per_s": tokens / ((qk_ms + pv_ms) * 1e-3)}


def speculative_record(pk, dev, peak, bits=4, S=4):
    """Several queries per KV head: the GQA shape (32 query / 8 KV heads, 131k tokens)
    decoding S = 4 draft positions at once, i.e. 16 query rows per KV head (two
    launches of 8).  Per-launch-call times of q·Kᵀ, p·V and the fused attention over
    the whole cache; tokens/s counts cache tokens x draft positions."""
    import torch
    w0 = synth.WORKLOADS[2]
    w = synth.Workload(w0.name + " x4 draft positions", w0.batch, w0.q_heads * S, w0.kv_heads, w0.seq,
                       (bits,), w0.seed)
    rec = workload_record(pk, dev, 2, bits, peak, w_override=w)
    rec["workload"] = f"speculative: gqa8b b1 hkv8 d128 seq131072, {S} draft positions x G=4 (16 rows per kv head)"
    rec["tokens_per_s_x_positions"] = rec["step_tokens_per_s"] * S
    return rec


# ------------------------------------------------------------------ the CUDA path: the run
def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from decode_gemv_packkv_b200 import packkv as pk

    w0 = synth.WORKLOADS[args.workload]
    w = synth.Workload(w0.name, w0.batch, w0.q_heads, w0.kv_heads, w0.seq, w0.bits, rank_seed(w0.seed, rank))
    bits = args.bits or w.bits[0]
    B, Hq, Hkv, T = w.batch, w.q_heads, w.kv_heads, w.seq
    nb = T // 128
    kd, vd = upload(w, T, dev, structured=args.structured)

    # encoder throughput (prefill of the whole cache; fp16 bytes in)
    enc_cache = pk.PackKVCache(B, Hkv, nb, bits)
    for _ in range(2):
        pk.packkv_cache_reset(enc_cache)
        pk.packkv_encode_block(enc_cache, kd, vd, nb)
    n_enc = 3

    def encodes():
        for _ in range(n_enc):
            pk.packkv_cache_reset(enc_cache)
            pk.packkv_encode_block(enc_cache, kd, vd, nb)
    enc_ms = timed_ms(dev, encodes) / n_enc
    del enc_cache

    # R cache copies, together larger than L2
    cs1 = CacheSet(pk, dev, w, bits, kd, vd, R=1)
    per_copy = cs1.k_used + cs1.v_used + 2 * cs1.index_bytes
    R = max(3, int(np.ceil(2.5 * L2_BYTES / per_copy)))
    del cs1
    cs = CacheSet(pk, dev, w, bits, kd, vd, R=R)

    g_step = cs.graph("qk", "pv")
    # exactly K timed and W warm-up steps: whole rotations, then the first steps of one more
    K = max(1, args.steps)
    W = max(1, args.warmup)
    partial = {n: cs.graph("qk", "pv", n=n) for n in {K % R, W % R} if n}

    def run_steps(n):
        for _ in range(n // R):
            g_step.replay()
        if n % R:
            partial[n % R].replay()

    run_steps(W)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(physical_gpu_index(dev.index))
    if rank == 0:
        sampler.start()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ms = timed_ms(dev, lambda: run_steps(K), pre_sleep=False)
    barrier(dev)
    clocks = sampler.stop() if rank == 0 else None
    ms = max_over_ranks(ms, dev)
    ms_per_step = ms / K

    # per-kernel durations (each kernel alone, same rotation), for the roofline
    qk_ms = cs.per_launch_ms("qk", min_launches=max(60, K))
    pv_ms = cs.per_launch_ms("pv", min_launches=max(60, K))
    attn_ms = cs.per_launch_ms("attn", min_launches=max(60, K))
    qk_bytes, pv_bytes, attn_bytes = cs.bytes()
    hbm_peak, peak_note = measured_peaks()
    qk_gbs = qk_bytes / (qk_ms * 1e-3) / 1e9
    pv_gbs = pv_bytes / (pv_ms * 1e-3) / 1e9
    dom = "qk" if qk_ms >= pv_ms else "pv"
    dom_gbs, dom_bytes, dom_ms = (qk_gbs, qk_bytes, qk_ms) if dom == "qk" else (pv_gbs, pv_bytes, pv_ms)
    fp16_bytes = cs.fp16_bytes

    # cuBLAS fp16 GEMV on the uncompressed cache (the comparison the pages make)
    cb_qk, cb_pv = cublas_ms(dev, kd, vd, Hq // Hkv)

    # end to end through the public API: pinned host q -> device, q·Kᵀ, softmax (caller's
    # step between the products), p·V, out -> pinned host; every step synchronised
    q_host = torch.from_numpy(synth.queries(w, 0)).pin_memory()
    out_host = torch.empty((B, Hq, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(cs.q[0])
    p_e2e = torch.zeros((B, Hq, cs.ld), dtype=torch.float32, device=dev)

    def e2e_step(i):
        q_dev.copy_(q_host, non_blocking=True)
        pk.packkv_qk_gemv(cs.caches[i], q_dev, SCALE, cs.scores[i])
        p_e2e[:, :, :T] = torch.softmax(cs.scores[i][:, :, :T], dim=-1)
        pk.packkv_pv_gemv(cs.caches[i], p_e2e, cs.outs[i], cs.ws[i])
        out_host.copy_(cs.outs[i], non_blocking=True)

    for i in range(3):
        e2e_step(i % R)
    torch.cuda.synchronize(dev)
    n_e2e = max(30, min(1000, args.steps // 10))

    def e2e_time(one_step):
        barrier(dev)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record()
        for i in range(n_e2e):
            one_step(i)
            torch.cuda.current_stream(dev).synchronize()
        b_.record()
        torch.cuda.synchronize(dev)
        return max_over_ranks(a_.elapsed_time(b_), dev) / n_e2e

    e2e_eager_ms = e2e_time(lambda i: e2e_step(i % R))
    # the same step captured once per cache copy in a CUDA graph (the calls make no
    # allocation and no synchronisation, so a serving loop can replay them); every
    # replay still copies q in from pinned memory and the output back out
    e2e_graphs = [capture(dev, lambda i=i: e2e_step(i)) for i in range(R)]
    for g in e2e_graphs:
        g.replay()
    torch.cuda.synchronize(dev)
    e2e_ms = e2e_time(lambda i: e2e_graphs[i % R].replay())
    comp = compression_entry(cs, bits)
    comp["raw_fraction_k"] = comp["raw_share_k"]

    result = {
        "metric": METRIC, "value": job_value(world, B * T, ms_per_step), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8xs8->s32 (tensor cores) + f32",
        "data": ("synthetic, run-structured (few levels per channel held for random runs)" if args.structured else
                 "synthetic (seeded; K per-channel N(mu,sigma) with outlier channels, V N(0,1)); no weights needed"),
        "config": {"workload": w0.name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": 128, "seq": T,
                   "bits": bits, "block_tokens": 128, "group_tokens": 32, "reorder_key": "k-code-sum",
                   "l2": f"inputs larger than L2: steps rotate over {R} packed-cache copies "
                         f"({R * per_copy / 1e6:.0f} MB) with their own q and p",
                   "step": "packkv_qk_gemv + packkv_pv_gemv over every sequence and head",
                   "timing": "CUDA graph of R steps replayed; CUDA events on the launching stream",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "qk": gemv_entry(qk_ms, cs.k_used + cs.index_bytes, qk_bytes, fp16_bytes, B * T, hbm_peak),
        "pv": gemv_entry(pv_ms, cs.v_used + cs.index_bytes, pv_bytes, fp16_bytes, B * T, hbm_peak),
        "fused_attention": {"ms": attn_ms, "bytes": attn_bytes, "gbs": attn_bytes / (attn_ms * 1e-3) / 1e9,
                            "frac_hbm": attn_bytes / (attn_ms * 1e-3) / 1e9 / hbm_peak,
                            "tokens_per_s": world * B * T / (attn_ms * 1e-3), "speedup_vs_step": ms_per_step / attn_ms,
                            "call": "packkv_attention_decode: q·Kᵀ, online softmax and p·V in one pass"},
        "cublas_fp16": {"qk_ms": cb_qk, "pv_ms": cb_pv, "qk_speedup": cb_qk / qk_ms, "pv_speedup": cb_pv / pv_ms,
                        "qk_gbs": fp16_bytes / (cb_qk * 1e-3) / 1e9, "pv_gbs": fp16_bytes / (cb_pv * 1e-3) / 1e9},
        "encode": {"ms": enc_ms, "fp16_in_gbs": 2 * fp16_bytes / (enc_ms * 1e-3) / 1e9,
                   "blocks_per_s": 2 * B * Hkv * nb / (enc_ms * 1e-3),
                   "bytes_per_launch": 2 * fp16_bytes + cs.k_used + cs.v_used,
                   "frac_hbm": (2 * fp16_bytes + cs.k_used + cs.v_used) / (enc_ms * 1e-3) / 1e9 / hbm_peak},
        "compression": comp,
        "roofline": {"bound": "hbm", "kernel": "packkv_qk_gemv" if dom == "qk" else "packkv_pv_gemv",
                     "achieved": dom_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": dom_gbs / hbm_peak,
                     "traffic": DRAM_TRAFFIC.get((w0.name, bits, dom)),
                     "traffic_note": "first-pass kernel DRAM read+write per launch (ncu), null when the kernel "
                                     "changed after the capture",
                     "algorithmic_bytes_per_launch": dom_bytes, "launch_ms": dom_ms,
                     "frac_compressed_bytes": (cs.k_used if dom == "qk" else cs.v_used) / (dom_ms * 1e-3) / 1e9
                     / hbm_peak,
                     "peak_source": peak_note},
        "e2e": {"value": job_value(world, B * T, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(q_host.numel() * 2), "d2h_bytes_per_step": int(out_host.numel() * 4),
                "note": "per step: pinned q H2D, packkv_qk_gemv, softmax (torch, the caller's step), "
                        "packkv_pv_gemv, out D2H, then a host sync; the step's calls replayed as a CUDA graph",
                "eager_ms_per_step": e2e_eager_ms,
                "eager_value": job_value(world, B * T, e2e_eager_ms)},
        "gpu_launches": KERNELS_PER_STEP * K,
        "clocks": clocks,
    }
    del cs, e2e_graphs, g_step, partial
    torch.cuda.empty_cache()
    if not args.no_sub:
        subs = []
        t_sub = time.time()
        subs.append(workload_record(pk, dev, 0, 4, hbm_peak))
        kd1, vd1 = upload(synth.WORKLOADS[1], synth.WORKLOADS[1].seq, dev, structured=True)
        for b in (4, 2):
            subs.append(workload_record(pk, dev, 1, b, hbm_peak, structured=True, kd=kd1, vd=vd1))
        del kd1, vd1
        w2 = synth.WORKLOADS[2]
        kd2, vd2 = upload(w2, w2.seq, dev)
        for b in (4, 2):
            subs.append(workload_record(pk, dev, 2, b, hbm_peak, kd=kd2, vd=vd2))
        del kd2, vd2
        torch.cuda.empty_cache()
        subs.append(workload_record(pk, dev, 3, 3, hbm_peak))
        torch.cuda.empty_cache()
        subs.append(ragged_record(pk, dev, hbm_peak))
        torch.cuda.empty_cache()
        subs.append(speculative_record(pk, dev, hbm_peak))
        torch.cuda.empty_cache()
        for b in (2, 3, 4):
            subs.append(streaming_record(pk, dev, b))
            torch.cuda.empty_cache()
        result["workloads"] = subs
        result["workloads_seconds"] = time.time() - t_sub
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w0, bits, budget_s=args.cpu_seconds)
    if world > 1:
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------------------ the CPU oracle (baseline / reference arm)
def oracle_step_sample(w, bits, n_blocks, head=0):
    """A sample of the workload for the oracle: n_blocks of sequence (0, head)."""
    import oracle as O
    ks, vs = synth.kv_slice(w.seed, w.kv_heads, 0, head % w.kv_heads, n_blocks * 128)
    cache = O.OracleCache(1, 1, n_blocks, bits)
    cache.encode_blocks(ks[None, None], vs[None, None], n_blocks)
    q = synth.queries(w)[:1, :w.group]
    return cache, q


def oracle_gemv_seconds(cache, q):
    """One oracle pass of the step on a sample: q·Kᵀ then p·V (decoding the records)."""
    import oracle as O
    cache._decoded.clear()           # time the decode too, as the GPU step does
    t0 = time.perf_counter()
    scores, _ = O.cache_qk(cache, q, SCALE)
    O.cache_pv(cache, O.softmax(scores))
    return time.perf_counter() - t0


def oracle_worker(job):
    """One host core: repeat the oracle step on its own sample for `budget` seconds;
    returns (tokens, seconds)."""
    wid, bits, n_blocks, head, budget = job
    w = synth.WORKLOADS[wid]
    cache, q = oracle_step_sample(w, bits, n_blocks, head)
    tok, secs = 0, 0.0
    while secs < budget or tok == 0:
        secs += oracle_gemv_seconds(cache, q)
        tok += n_blocks * 128
    return tok, secs


def _wid_of(w):
    return next(i for i, x in synth.WORKLOADS.items() if x.name == w.name)


def cpu_baseline(w, bits, budget_s=15.0):
    """The oracle timed on the host cores: one core, then every core (one process each,
    spawned, each on its own (sequence, kv head) sample).  A whole-workload token needs
    all kv heads, so sample tokens count 1/kv_heads each."""
    import multiprocessing as mp
    wid = _wid_of(w)
    tok1, sec1 = oracle_worker((wid, bits, 16, 0, budget_s))
    one = tok1 / sec1 / w.kv_heads
    cores = os.cpu_count() or 1
    ctx = mp.get_context("spawn")
    t0 = time.perf_counter()
    with ctx.Pool(cores) as pool:
        res = pool.map(oracle_worker, [(wid, bits, 16, i, budget_s) for i in range(cores)])
    wall = time.perf_counter() - t0
    tot = sum(r[0] for r in res)
    span = max(r[1] for r in res)
    allc = tot / span / w.kv_heads
    return {"value": allc, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"per core one (sequence, kv head) x 16 blocks (2048 tokens) of the workload "
                      f"(G={w.group} query heads), q·Kᵀ + softmax + p·V incl. record decoding, repeated for "
                      f"{budget_s:.0f} s; sample tokens count 1/{w.kv_heads} of a workload token",
            "seconds": span, "wall_seconds": wall,
            "single_core": {"value": one, "cores": 1, "seconds": sec1}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    bits = args.bits or w.bits[0]
    # size each step's sample so that warmup + steps take a few minutes at most
    cache, q = oracle_step_sample(w, bits, 1)
    one = oracle_gemv_seconds(cache, q)
    n_blocks = int(max(1, min(64, REFERENCE_SECONDS / max(1, args.steps + args.warmup) / max(one, 1e-4))))
    cache, q = oracle_step_sample(w, bits, n_blocks)
    for _ in range(args.warmup):
        oracle_gemv_seconds(cache, q)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_gemv_seconds(cache, q)
    step_s = total / args.steps
    # one sample step decodes n_blocks*128 tokens of one kv head: 1/kv_heads of a workload token each
    value = n_blocks * 128 / step_s / w.kv_heads
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": step_s * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": w.name, "bits": bits},
           "step": f"the CPU oracle on a sample: {n_blocks} block(s) ({n_blocks * 128} tokens) of one kv head "
                   f"(G={w.group} query heads), q·Kᵀ + softmax + p·V including record decoding; ms_per_step is "
                   "the time of that sample step",
           "whole_workload_ms_per_step_extrapolated": 1e3 * w.batch * w.seq / value,
           "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": UNIT,
                            "sample": f"{n_blocks} block(s) of one kv head per step; tokens count 1/{w.kv_heads}"},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=300)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=1, help="workload id (synth.WORKLOADS)")
    ap.add_argument("--bits", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="headline workload only (no per-workload sub-records)")
    ap.add_argument("--structured", action="store_true",
                    help="run-structured inputs for the headline workload (compressed records; profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
