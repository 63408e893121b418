"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare.

Acceptance (packed-cache format v1, section 7): encoder output bit-exact; scores and outputs
within 1e-3 * sum|terms| per element (exact 0 where sum|terms| = 0).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

TOL = 1e-3


def assert_within_terms(gpu: np.ndarray, ref: np.ndarray, abs_terms: np.ndarray, what: str):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    bound = TOL * abs_terms
    bad = ~(err <= bound)
    zero = abs_terms == 0
    bad |= zero & (gpu != 0)
    if np.any(bad):
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, e.g. "
                             + ", ".join(f"{tuple(i)}: gpu={gpu[tuple(i)]:.9g} ref={ref[tuple(i)]:.9g} "
                                         f"bound={bound[tuple(i)]:.3g}" for i in idx))
    if err.size == 0:
        return 0.0
    return float(np.max(np.where(abs_terms > 0, err / np.maximum(abs_terms, 1e-300), 0.0)))


def gpu_records(cache, which: str):
    """(arena bytes used, index int64 [B,H,nb,2]) copied back from the device."""
    arena = (cache.k_arena if which == "k" else cache.v_arena).cpu().numpy()
    index = (cache.k_index if which == "k" else cache.v_index).cpu().numpy().view(np.uint32).astype(np.int64)
    return arena, index


def gpu_record(arena: np.ndarray, index: np.ndarray, b: int, h: int, i: int) -> bytes:
    off, ln = index[b, h, i]
    return bytes(arena[off * 16:(off + ln) * 16])


def compare_encoder(cache, ocache: O.OracleCache, full_layout: bool = True, blocks=None):
    """Bit-exact comparison of records, index, arena ends and permutations."""
    for which in ("k", "v"):
        arena, index = gpu_records(cache, which)
        o_index = ocache.k_index if which == "k" else ocache.v_index
        nb = ocache.n_blocks
        for b in range(ocache.batch):
            for h in range(ocache.kv_heads):
                for i in range(nb):
                    if blocks is not None and (b, h, i) not in blocks:
                        continue
                    got = gpu_record(arena, index, b, h, i)
                    want = ocache.record(which, b, h, i)
                    if got != want:
                        diff = next(j for j in range(min(len(got), len(want))) if got[j] != want[j]) \
                            if len(got) == len(want) else -1
                        raise AssertionError(f"{which} record ({b},{h},{i}) differs: len {len(got)} vs "
                                             f"{len(want)}, first differing byte {diff}")
        if full_layout:
            assert np.array_equal(index[:, :, :nb], o_index[:, :, :nb].astype(np.int64)), f"{which} index"
            ends = cache.ctrl.cpu().numpy()
            assert ends[0 if which == "k" else 1] * 16 == len(ocache.k_arena if which == "k" else ocache.v_arena)
    if cache.perm is not None:
        perm = cache.perm.cpu().numpy()
        for b in range(ocache.batch):
            for h in range(ocache.kv_heads):
                for i in range(ocache.n_blocks):
                    if blocks is not None and (b, h, i) not in blocks:
                        continue
                    assert np.array_equal(perm[b, h, i], ocache.perm[b, h, i]), f"perm ({b},{h},{i})"


def to_dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()
