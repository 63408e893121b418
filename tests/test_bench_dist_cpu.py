"""The multi-GPU plumbing of bench.py, exercised with two gloo ranks on the CPU.

With N > 1 every rank decodes its own batch (independent problems: weak
scaling, no collective on the data path).  The only collectives are the
barrier around the timed region and the max of the step times over ranks;
the job throughput is the tokens of all ranks over that max.
"""
import json
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

import bench
from decode_gemv_packkv_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        bench.barrier(None)
        # rank r "measured" (r + 1) * 1.5 ms: every rank must see the slowest
        slowest = bench.max_over_ranks((rank + 1) * 1.5)
        wl = synth.WORKLOADS[0]
        seed = bench.rank_seed(wl.seed, rank)
        ks, vs = synth.kv_slice(seed, wl.kv_heads, 0, 0, 256)
        digest = float(np.float64(ks.astype(np.float64).sum() + 3 * vs.astype(np.float64).sum()))
        bench.barrier(None)
        q.put({"rank": rank, "env": [r, w, local], "slowest": slowest, "seed": seed, "digest": digest})
    finally:
        dist.destroy_process_group()


def _run_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out, key=lambda d: d["rank"])


def test_two_gloo_ranks_agree_on_the_slowest_step_and_decode_distinct_batches():
    res = _run_ranks(2)
    assert [d["env"] for d in res] == [[0, 2, 0], [1, 2, 1]]
    assert all(d["slowest"] == 3.0 for d in res)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["digest"] != res[1]["digest"]          # weak scaling: each rank its own synthetic batch


def test_job_value_counts_every_rank_over_the_max_time():
    # 2 ranks x 32768 tokens in a 0.1 ms step -> 655.36 M tokens/s
    assert bench.job_value(2, 32768, 0.1) == pytest.approx(655.36e6)
    assert bench.job_value(1, 32768, 0.1) == pytest.approx(327.68e6)


def test_single_process_helpers_are_identities():
    assert bench.max_over_ranks(2.5) == 2.5
    bench.barrier(None)                                  # no process group: a no-op


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_reference_arm_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(bench, "REFERENCE_SECONDS", 2.0)
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "0"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_median_ms_takes_the_median_of_five_timings(monkeypatch):
    """Sub-record kernel times are the median of five CUDA-event timings."""
    import bench
    seq = iter([5.0, 1.0, 9.0, 3.0, 7.0])
    calls = []
    monkeypatch.setattr(bench, "timed_ms", lambda dev, fn: calls.append(fn) or next(seq))
    assert bench.median_ms(None, "f") == 5.0
    assert calls == ["f"] * 5
