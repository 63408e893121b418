"""Encoder ablation on one GPU: reorder key x unit mode x code width x input kind.

For each combination (every reorder key with frame-of-reference units, and the
default key with width-only units) this encodes a (1 sequence x H heads x T tokens) cache and
reports the K and V compression ratios (fp16 bytes / (record + index bytes); plain
b-bit quantization, codes plus fp16 min and scale, for comparison), the share of
blocks stored raw, and the CUDA-event time of one packkv_qk_gemv and one
packkv_pv_gemv launch over the whole cache.  Inputs are the seeded synthetic
generators of `synth` (the 32-head 32k-token workload's distributions by default);
"structured" inputs hold few levels per channel for random run lengths, so that the
frame-of-reference units of the packed format get narrow and compressed records
appear (PackKV paper page, Figure 2: the token reorder is meant to help the
channel-direction packing that follows it).  Several cache copies, together larger
than L2, are rotated so that every launch reads HBM.

    python -m decode_gemv_packkv_b200.ablation [--heads 32] [--tokens 32768]

prints one JSON line per (input kind, bits, reorder key, unit mode).
"""
import argparse
import json

import numpy as np
import torch

from . import packkv as pk
from . import synth

L2_BYTES = 126 * 1024 * 1024
KEYS = {"identity": pk.KEY_IDENTITY, "k-code-sum": pk.KEY_K_SUM, "kv-code-sum": pk.KEY_KV_SUM}


def _inputs(heads: int, tokens: int, structured: bool, seed: int, dev):
    k = torch.empty((1, heads, tokens, synth.HEAD_DIM), dtype=torch.float16, device=dev)
    v = torch.empty_like(k)
    for h in range(heads):
        ks, vs = synth.kv_slice(seed, heads, 0, h, tokens, structured=structured)
        k[0, h].copy_(torch.from_numpy(ks))
        v[0, h].copy_(torch.from_numpy(vs))
    return k, v


def _raw_share(cache: pk.PackKVCache, bits: int) -> tuple[float, float]:
    raw16 = pk.record_bytes_max(bits) // 16
    nb = cache.n_blocks
    k = cache.k_index[..., :nb, 1].cpu()
    v = cache.v_index[..., :nb, 1].cpu()
    return float((k == raw16).float().mean()), float((v == raw16).float().mean())


def _time(fn, copies: int, reps: int) -> float:
    """Microseconds per launch: one CUDA graph holds one call per cache copy and is
    replayed (no host launch overhead between the timed kernels)."""
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(copies):  # warm-up, and the workspaces are allocated before capture
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(copies):
                fn(i)
        for _ in range(3):
            g.replay()
        n = max(1, reps // copies)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (n * copies)


def run(heads: int, tokens: int, bits_list, reps: int, seed: int):
    if not torch.cuda.is_available():
        raise RuntimeError("the ablation runs the CUDA kernels and needs a GPU")
    dev = torch.device("cuda", 0)
    nb = tokens // 128
    T = nb * 128
    fp16_bytes = heads * T * 128 * 2
    index_bytes = heads * nb * 8
    q = torch.from_numpy(synth.queries(synth.Workload("ablation", 1, heads, heads, T, (4,), seed), 0)).to(dev)
    scores = torch.empty((1, heads, T), dtype=torch.float32, device=dev)
    p = torch.softmax(torch.randn((1, heads, T), device=dev), dim=-1).contiguous()
    out = torch.empty((1, heads, 128), dtype=torch.float32, device=dev)
    scale = 1.0 / np.sqrt(128.0)
    for kind in ("iid", "structured"):
        kd, vd = _inputs(heads, T, kind == "structured", seed, dev)
        for bits in bits_list:
            # every reorder key with frame-of-reference units, then width-only units (base
            # 0) with the default key: the width-only variant of the packing
            combos = [(kn, kv, "frame-of-reference", pk.UNITS_FOR) for kn, kv in KEYS.items()]
            combos.append(("k-code-sum", pk.KEY_K_SUM, "width-only", pk.UNITS_WIDTH_ONLY))
            for key_name, key, unit_name, unit_mode in combos:
                first = pk.PackKVCache(1, heads, nb, bits, reorder_key=key, unit_mode=unit_mode)
                pk.packkv_encode_block(first, kd, vd, nb)
                k_used, v_used = first.arena_used()
                raw_k, raw_v = _raw_share(first, bits)
                copies = max(3, int(np.ceil(2.5 * L2_BYTES / (k_used + v_used + 2 * index_bytes))))
                caches = [first]
                for _ in range(copies - 1):
                    c = pk.PackKVCache(1, heads, nb, bits, reorder_key=key, arena_bytes=max(k_used, v_used) + 16,
                                       unit_mode=unit_mode)
                    pk.packkv_encode_block(c, kd, vd, nb)
                    caches.append(c)
                qk_us = _time(lambda i: pk.packkv_qk_gemv(caches[i], q, scale, scores), copies, reps)
                pv_us = _time(lambda i: pk.packkv_pv_gemv(caches[i], p, out), copies, reps)
                bad = [pk.packkv_get_status(c) for c in caches if pk.packkv_get_status(c) != 0]
                print(json.dumps({
                    "inputs": kind, "bits": bits, "reorder_key": key_name, "units": unit_name, "heads": heads,
                    "tokens": T,
                    "cr_k": fp16_bytes / (k_used + index_bytes), "cr_v": fp16_bytes / (v_used + index_bytes),
                    "plain_quant_cr": 128 * 128 * 2 / (128 * 128 * bits / 8 + 512),  # codes + fp16 min/scale
                    "raw_share_k": raw_k, "raw_share_v": raw_v,
                    "qk_us": qk_us, "pv_us": pv_us,
                    "qk_gbs": (k_used + index_bytes + heads * T * 4) / qk_us * 1e-3,
                    "pv_gbs": (v_used + index_bytes + heads * T * 4) / pv_us * 1e-3,
                    "status": bad[0] if bad else 0}), flush=True)
                del caches, first
        del kd, vd
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--heads", type=int, default=32)
    ap.add_argument("--tokens", type=int, default=32768)
    ap.add_argument("--bits", type=int, nargs="+", default=[2, 3, 4])
    ap.add_argument("--reps", type=int, default=60)
    ap.add_argument("--seed", type=int, default=1001)
    a = ap.parse_args()
    run(a.heads, a.tokens, a.bits, a.reps, a.seed)


if __name__ == "__main__":
    main()
