"""Seeded synthetic inputs for the PackKV decode path.

This module only draws random numbers; it holds none of the method's arithmetic
(no quantization, packing or products), so both the CPU oracle's tests and the
CUDA path's tests and benchmark may use it.

Distributions (the workloads the PackKV pages measure on are LLM KV caches; no
trained weights or datasets are available, so these stand in for them):
  * K[t, c] = mu_c + sigma_c * N(0, 1) with mu_c ~ N(0, 1), sigma_c ~ U(0.5, 2)
    and 4 outlier channels per (batch, head) whose sigma is multiplied by 10.
  * V[t, c] ~ N(0, 1).   q ~ N(0, 1), one vector per query head.
  * Every draw is fp32 from numpy's PCG64, rounded to fp16 (round to nearest).
  * Sequence (b, h) of a config with seed s uses PCG64(s).jumped(b * Hkv + h),
    so large configs can be generated slice by slice with bounded host memory.
  * q uses PCG64(s + 1) and p (for timing-only runs) PCG64(s + 2).
A "structured" variant draws K and V from a few levels per channel with runs of
repeated values, so that pack units get every width 0..b (compressed records).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    seq: int
    bits: tuple
    seed: int
    decode_steps: int = 0       # streaming growth: tokens seq .. seq+decode_steps-1 are appended one by one

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads


# The five workloads the PackKV decode path is measured on (shapes, bits, seeds).
WORKLOADS = {
    0: Workload("single-head b1 h1 d128 seq4096 4-bit", 1, 1, 1, 4096, (4,), 1000),
    1: Workload("llama7b-decode mha b1 h32 d128 seq32768 4-bit", 1, 32, 32, 32768, (4,), 1001),
    2: Workload("gqa8b b1 hq32 hkv8 d128 seq131072 4/2-bit", 1, 32, 8, 131072, (4, 2), 1002),
    3: Workload("batched b16 h32 d128 seq16384 3-bit", 16, 32, 32, 16384, (3,), 1003),
    4: Workload("streaming b4 h32 d128 prefill8192+4096 steps", 4, 32, 32, 8192, (2, 3, 4), 1004,
                decode_steps=4096),
}


def _slice_rng(seed: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed).jumped(index))


def kv_slice(seed: int, kv_heads: int, b: int, h: int, tokens: int, start: int = 0,
             structured: bool = False):
    """K, V for one (batch, kv-head) sequence: fp16 [tokens, 128] each.

    `start` skips the first `start` tokens of the same sequence (draws are made
    for all tokens up to start + tokens, in token order, so a sequence is the
    same whether generated at once or in pieces).
    """
    rng = _slice_rng(seed, b * kv_heads + h)
    mu = rng.standard_normal(HEAD_DIM, dtype=np.float32)
    sigma = rng.uniform(0.5, 2.0, HEAD_DIM).astype(np.float32)
    outliers = rng.choice(HEAD_DIM, 4, replace=False)
    sigma[outliers] *= np.float32(10.0)
    n = start + tokens
    if not structured:
        zk = rng.standard_normal((n, HEAD_DIM), dtype=np.float32)
        zv = rng.standard_normal((n, HEAD_DIM), dtype=np.float32)
    else:
        # few levels per channel, held for random run lengths: pack units of
        # width 0..4 all occur; some channels are constant
        levels = rng.integers(1, 17, HEAD_DIM)
        runs = rng.integers(1, 48, (n, HEAD_DIM))
        zk = np.empty((n, HEAD_DIM), np.float32)
        zv = np.empty((n, HEAD_DIM), np.float32)
        for z in (zk, zv):
            draw = rng.integers(0, 1 << 30, (n, HEAD_DIM)) % levels[None, :]
            hold = (np.arange(n)[:, None] % runs[0][None, :]) != 0
            # each held position repeats the draw of the last position not held
            src = np.where(hold, 0, np.arange(n)[:, None])
            src = np.maximum.accumulate(src, axis=0)
            draw = np.take_along_axis(draw, src, axis=0)
            z[:] = (draw.astype(np.float32) - levels[None, :] / 2.0) / 4.0
    k = (mu[None, :] + sigma[None, :] * zk[start:]).astype(np.float16)
    v = zv[start:].astype(np.float16)
    return k, v


def kv_cache_inputs(w: Workload, tokens: int | None = None, structured: bool = False):
    """Full K, V [B, Hkv, tokens, 128] fp16 for a workload (host memory!)."""
    t = w.seq if tokens is None else tokens
    k = np.empty((w.batch, w.kv_heads, t, HEAD_DIM), np.float16)
    v = np.empty_like(k)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            k[b, h], v[b, h] = kv_slice(w.seed, w.kv_heads, b, h, t, structured=structured)
    return k, v


def queries(w: Workload, step: int = 0) -> np.ndarray:
    """q [B, Hq, 128] fp16 for decode step `step`."""
    rng = _slice_rng(w.seed + 1, step)
    return rng.standard_normal((w.batch, w.q_heads, HEAD_DIM), dtype=np.float32).astype(np.float16)


def timing_probs(w: Workload, tokens: int) -> np.ndarray:
    """Any nonnegative p [B, Hq, tokens] fp32 summing to 1 per row (timing runs only)."""
    rng = _slice_rng(w.seed + 2, 0)
    p = rng.random((w.batch, w.q_heads, tokens), dtype=np.float32)
    return (p / p.sum(axis=-1, keepdims=True)).astype(np.float32)


def small_case(seed: int, batch: int, kv_heads: int, group: int, tokens: int,
               structured: bool = False):
    """A small arbitrary-shape case for tests: (k, v, q) with k, v [B, Hkv, T, 128]."""
    k = np.empty((batch, kv_heads, tokens, HEAD_DIM), np.float16)
    v = np.empty_like(k)
    for b in range(batch):
        for h in range(kv_heads):
            k[b, h], v[b, h] = kv_slice(seed, kv_heads, b, h, tokens, structured=structured)
    rng = _slice_rng(seed + 1, 0)
    q = rng.standard_normal((batch, kv_heads * group, HEAD_DIM), dtype=np.float32).astype(np.float16)
    return k, v, q
