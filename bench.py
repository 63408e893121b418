"""Benchmark of the PackKV decode path on B200: fused unpack + GEMV throughput.

One step = packkv_qk_gemv then packkv_pv_gemv over the whole packed cache of
the workload (every sequence and head), i.e. the two decode-time products of
the PackKV pages (Figure 1 attention, Figure 2 fused decompression + GEMV).
Default workload: Llama-7B-style decode layer, 32 MHA heads, head_dim 128,
batch 1, 32768 cached tokens, 4-bit codes (synthetic K/V with the per-channel
outlier distribution; see decode_gemv_packkv_b200/synth.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Timing: W untimed steps, then K steps bracketed
by a barrier and a device synchronize, CUDA events on the launching stream,
max over ranks.  Inputs exceed L2: steps rotate over several cache copies.
--impl reference times the CPU oracle on a bounded sample of the same workload.
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
# one capture of the 32-head 32k-token 4-bit cache; summary in profiles/).  None for
# other workloads; to be re-measured whenever the kernel changes.
DRAM_TRAFFIC = {("llama7b-decode mha b1 h32 d128 seq32768 4-bit", 4): 75.735808e6 + 1.264384e6}


# ------------------------------------------------------------------ the CUDA path
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
    # K/V generated per slice on the host, encoded on the device into R copies of the cache
    kd = torch.empty((B, Hkv, T, 128), dtype=torch.float16, device=dev)
    vd = torch.empty_like(kd)
    for b in range(B):
        for h in range(Hkv):
            ks, vs = synth.kv_slice(w.seed, Hkv, b, h, T)
            kd[b, h].copy_(torch.from_numpy(ks))
            vd[b, h].copy_(torch.from_numpy(vs))
    stream = torch.cuda.current_stream(dev)

    # encoder throughput (prefill of the whole cache; fp16 bytes in)
    enc_cache = pk.PackKVCache(B, Hkv, nb, bits)
    for _ in range(2):
        pk.packkv_cache_reset(enc_cache)
        pk.packkv_encode_block(enc_cache, kd, vd, nb)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_enc = 3
    e0.record(stream)
    for _ in range(n_enc):
        pk.packkv_cache_reset(enc_cache)
        pk.packkv_encode_block(enc_cache, kd, vd, nb)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    enc_ms = e0.elapsed_time(e1) / n_enc
    k_used, v_used = enc_cache.arena_used()
    index_bytes = B * Hkv * nb * 8
    fp16_bytes = B * Hkv * T * 128 * 2
    raw_bytes = B * Hkv * nb * pk.record_bytes_max(bits)
    del enc_cache

    # R cache copies, together larger than L2
    per_copy = k_used + v_used + 2 * index_bytes
    R = max(3, int(np.ceil(2.5 * L2_BYTES / per_copy)))
    caches = []
    for _ in range(R):
        c = pk.PackKVCache(B, Hkv, nb, bits, arena_bytes=max(k_used, v_used) + 16)
        pk.packkv_encode_block(c, kd, vd, nb)
        caches.append(c)
    assert all(pk.packkv_get_status(c) == 0 for c in caches)
    q = [torch.from_numpy(synth.queries(w, i)).to(dev) for i in range(R)]
    ld = (T + 3) // 4 * 4
    p_np = synth.timing_probs(w, T)
    p = []
    for i in range(R):
        t_ = torch.zeros((B, Hq, ld), dtype=torch.float32, device=dev)
        t_[:, :, :T] = torch.from_numpy(p_np).to(dev)
        p.append(t_)
    scores = [torch.empty((B, Hq, ld), dtype=torch.float32, device=dev) for _ in range(R)]
    outs = [torch.empty((B, Hq, 128), dtype=torch.float32, device=dev) for _ in range(R)]
    wss = [c.workspace(Hq) for c in caches]

    def step(i, do_qk=True, do_pv=True):
        if do_qk:
            pk.packkv_qk_gemv(caches[i], q[i], SCALE, scores[i])
        if do_pv:
            pk.packkv_pv_gemv(caches[i], p[i], outs[i], wss[i])

    # CUDA graphs: one graph = one step on each of n copies (launch overhead off the clock)
    def make_graph(do_qk, do_pv, n=R):
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for i in range(n):
                step(i, do_qk, do_pv)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                step(i, do_qk, do_pv)
        return g

    g_step, g_qk, g_pv = make_graph(True, True), make_graph(True, False), make_graph(False, True)
    # exactly K timed and W warm-up steps: whole rotations, then the first steps of one more
    K = max(1, args.steps)
    W = max(1, args.warmup)
    partial = {n: make_graph(True, True, n) for n in {K % R, W % R} if n}

    def run_steps(n):
        for _ in range(n // R):
            g_step.replay()
        if n % R:
            partial[n % R].replay()

    def timed(fn):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream(dev)
        a.record(cur)
        fn()
        b_.record(cur)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b_)

    run_steps(W)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(physical_gpu_index(dev.index))
    if rank == 0:
        sampler.start()
    barrier(dev)
    torch.cuda.synchronize(dev)
    ms = timed(lambda: run_steps(K))
    barrier(dev)
    clocks = sampler.stop() if rank == 0 else None
    ms = max_over_ranks(ms, dev)
    ms_per_step = ms / K

    # per-kernel durations (each kernel alone, same rotation), for the roofline
    reps = max(1, K // R)
    for g in (g_qk, g_pv):
        g.replay()

    def replays(g):
        for _ in range(reps):
            g.replay()

    qk_ms = timed(lambda: replays(g_qk)) / (reps * R)
    pv_ms = timed(lambda: replays(g_pv)) / (reps * R)

    # fused decode attention (one pass over both arenas; the scores never reach HBM)
    wsa = [c.attention_workspace(Hq) for c in caches]
    outs_a = [torch.empty((B, Hq, 128), dtype=torch.float32, device=dev) for _ in range(R)]

    def attn_graph():
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for i in range(R):
                pk.packkv_attention_decode(caches[i], q[i], SCALE, outs_a[i], wsa[i])
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(R):
                pk.packkv_attention_decode(caches[i], q[i], SCALE, outs_a[i], wsa[i])
        return g

    g_attn = attn_graph()
    g_attn.replay()
    attn_ms = timed(lambda: replays(g_attn)) / (reps * R)

    # algorithmic bytes per launch
    qk_bytes = k_used + index_bytes + B * Hq * 128 * 2 + B * Hq * T * 4
    pv_bytes = v_used + index_bytes + B * Hq * T * 4 + B * Hq * 128 * 4
    attn_bytes = k_used + v_used + 2 * index_bytes + B * Hq * 128 * 2 + B * Hq * 128 * 4
    hbm_peak, peak_note = measured_peaks()
    qk_gbs = qk_bytes / (qk_ms * 1e-3) / 1e9
    pv_gbs = pv_bytes / (pv_ms * 1e-3) / 1e9
    dom = "qk" if qk_ms >= pv_ms else "pv"
    dom_gbs, dom_bytes, dom_ms = (qk_gbs, qk_bytes, qk_ms) if dom == "qk" else (pv_gbs, pv_bytes, pv_ms)

    # cuBLAS fp16 GEMV on the uncompressed cache (the comparison the pages make)
    G = Hq // Hkv
    kf = kd.view(B * Hkv, T, 128)
    vf = vd.view(B * Hkv, T, 128)
    qh = torch.randn((B * Hkv, 128, G), dtype=torch.float16, device=dev)
    ph = torch.rand((B * Hkv, G, T), dtype=torch.float16, device=dev)
    for _ in range(3):
        torch.matmul(kf, qh)
        torch.matmul(ph, vf)
    torch.cuda.synchronize(dev)

    def time_fn(fn, n):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream(dev)
        a.record(cur)
        for _ in range(n):
            fn()
        b_.record(cur)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b_) / n

    n_cb = max(20, min(500, reps))
    cb_qk = time_fn(lambda: torch.matmul(kf, qh), n_cb)
    cb_pv = time_fn(lambda: torch.matmul(ph, vf), n_cb)

    # end to end through the public API: pinned host q -> device, q·Kᵀ, softmax (caller's
    # step between the products), p·V, out -> pinned host; every step synchronised
    q_host = torch.from_numpy(synth.queries(w, 0)).pin_memory()
    out_host = torch.empty((B, Hq, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(q[0])
    p_e2e = torch.zeros((B, Hq, ld), dtype=torch.float32, device=dev)

    def e2e_step(i):
        q_dev.copy_(q_host, non_blocking=True)
        pk.packkv_qk_gemv(caches[i], q_dev, SCALE, scores[i])
        p_e2e[:, :, :T] = torch.softmax(scores[i][:, :, :T], dim=-1)
        pk.packkv_pv_gemv(caches[i], p_e2e, outs[i], wss[i])
        out_host.copy_(outs[i], non_blocking=True)

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
    e2e_graphs = []
    s_cap = torch.cuda.Stream(dev)
    s_cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s_cap):
        e2e_step(0)
    torch.cuda.current_stream(dev).wait_stream(s_cap)
    torch.cuda.synchronize(dev)
    for i in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e2e_step(i)
        e2e_graphs.append(g)
    for i in range(R):
        e2e_graphs[i].replay()
    torch.cuda.synchronize(dev)
    e2e_ms = e2e_time(lambda i: e2e_graphs[i % R].replay())

    cr_k = fp16_bytes / (k_used + index_bytes)
    cr_v = fp16_bytes / (v_used + index_bytes)
    plain = 128 * 128 * 2 / (128 * 128 * bits / 8 + 512)
    result = {
        "metric": METRIC, "value": job_value(world, B * T, ms_per_step), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8xs8->s32 (tensor cores) + f32", "data": "synthetic (seeded; K per-channel N(mu,sigma) with outlier "
                                                       "channels, V N(0,1)); no weights needed",
        "config": {"workload": w0.name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": 128, "seq": T,
                   "bits": bits, "block_tokens": 128, "group_tokens": 32, "reorder_key": "k-code-sum",
                   "l2": f"inputs larger than L2: steps rotate over {R} packed-cache copies "
                         f"({R * per_copy / 1e6:.0f} MB) with their own q and p",
                   "step": "packkv_qk_gemv + packkv_pv_gemv over every sequence and head",
                   "timing": "CUDA graph of R steps replayed; CUDA events on the launching stream",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "qk": {"ms": qk_ms, "bytes": qk_bytes, "gbs": qk_gbs, "frac_hbm": qk_gbs / hbm_peak,
               "uncompressed_equiv_gbs": fp16_bytes / (qk_ms * 1e-3) / 1e9, "tokens_per_s": B * T / (qk_ms * 1e-3)},
        "pv": {"ms": pv_ms, "bytes": pv_bytes, "gbs": pv_gbs, "frac_hbm": pv_gbs / hbm_peak,
               "uncompressed_equiv_gbs": fp16_bytes / (pv_ms * 1e-3) / 1e9, "tokens_per_s": B * T / (pv_ms * 1e-3)},
        "fused_attention": {"ms": attn_ms, "bytes": attn_bytes, "gbs": attn_bytes / (attn_ms * 1e-3) / 1e9,
                            "frac_hbm": attn_bytes / (attn_ms * 1e-3) / 1e9 / hbm_peak,
                            "tokens_per_s": world * B * T / (attn_ms * 1e-3), "speedup_vs_step": ms_per_step / attn_ms,
                            "call": "packkv_attention_decode: q·Kᵀ, online softmax and p·V in one pass"},
        "cublas_fp16": {"qk_ms": cb_qk, "pv_ms": cb_pv, "qk_speedup": cb_qk / qk_ms, "pv_speedup": cb_pv / pv_ms,
                        "qk_gbs": fp16_bytes / (cb_qk * 1e-3) / 1e9, "pv_gbs": fp16_bytes / (cb_pv * 1e-3) / 1e9},
        "encode": {"ms": enc_ms, "fp16_in_gbs": 2 * fp16_bytes / (enc_ms * 1e-3) / 1e9,
                   "blocks_per_s": 2 * B * Hkv * nb / (enc_ms * 1e-3)},
        "compression": {"cr_k": cr_k, "cr_v": cr_v, "plain_quant_cr": plain,
                        "vs_plain_quant_k": cr_k / plain - 1, "vs_plain_quant_v": cr_v / plain - 1,
                        "raw_fraction_k": None if raw_bytes == 0 else k_used / raw_bytes},
        "roofline": {"bound": "hbm", "kernel": "packkv_qk_gemv" if dom == "qk" else "packkv_pv_gemv",
                     "achieved": dom_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": dom_gbs / hbm_peak,
                     "traffic": DRAM_TRAFFIC.get((w0.name, bits)) if dom == "pv" else None,
                     "traffic_note": "pv_kernel DRAM read+write per launch (ncu); pv_reduce_kernel adds the "
                                     "partials, which stay in L2",
                     "algorithmic_bytes_per_launch": dom_bytes, "launch_ms": dom_ms,
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
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w0, bits, budget_s=args.cpu_seconds)
    if world > 1:
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------------------ the CPU oracle (baseline / reference arm)
def oracle_step_sample(w, bits, n_blocks, seed_shift=0):
    """Builds a sample of the workload for the oracle: n_blocks of one (b, h) sequence."""
    import oracle as O
    ks, vs = synth.kv_slice(w.seed, w.kv_heads, 0, seed_shift % w.kv_heads, n_blocks * 128)
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


def cpu_baseline(w, bits, budget_s=15.0):
    cache, q = oracle_step_sample(w, bits, 16)
    secs = oracle_gemv_seconds(cache, q)
    tokens = 16 * 128
    total_t, total_tok = secs, tokens
    while total_t < budget_s:
        s = oracle_gemv_seconds(cache, q)
        total_t += s
        total_tok += tokens
    per_seq_head = total_tok / total_t
    # the workload processes all kv heads x G query heads; the oracle handles one kv head (G query heads)
    value = per_seq_head / (w.batch * w.kv_heads) if w.kv_heads else per_seq_head
    return {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"one kv head (G={w.group} query heads) x 16 blocks (2048 tokens) of the workload, "
                      f"q·Kᵀ + softmax + p·V incl. record decoding, repeated for {total_t:.1f} s; scaled to "
                      f"all {w.batch * w.kv_heads} (sequence, kv head) pairs",
            "seconds": total_t}


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
    tokens_per_s = n_blocks * 128 * args.steps / total / (w.batch * w.kv_heads)
    value = tokens_per_s
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * w.batch * w.seq / value,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": w.name, "bits": bits},
           "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": UNIT,
                            "sample": f"{n_blocks} block(s) of one kv head per step, scaled to the whole workload"},
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
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
