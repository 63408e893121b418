"""The encoder ablation tool on a small cache: i.i.d. inputs stay raw (the packed form
never beats plain b-bit codes there), structured inputs compress below plain
quantization size for every reorder key with frame-of-reference units, width-only
units are never smaller than those, and every call leaves the status clean."""
import contextlib
import io
import json

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_ablation_small_cache():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decode_gemv_packkv_b200 import ablation
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        ablation.run(heads=2, tokens=1024 + 77, bits_list=[2, 4], reps=6, seed=7)
    rows = [json.loads(line) for line in buf.getvalue().splitlines() if line.startswith("{")]
    assert len(rows) == 2 * 2 * 4
    by = {(r["inputs"], r["bits"], r["reorder_key"], r["units"]): r for r in rows}
    for r in rows:
        assert r["status"] == 0
        assert r["tokens"] == 1024
        assert r["qk_us"] > 0 and r["pv_us"] > 0
        if r["inputs"] == "iid":
            assert r["raw_share_k"] == 1.0 and r["raw_share_v"] == 1.0
            raw_cr = 128 * 128 * 2 / (528 + 2048 * r["bits"] + 8)  # raw record + index entry
            assert r["cr_k"] == pytest.approx(raw_cr, rel=1e-12) and r["cr_v"] == pytest.approx(raw_cr, rel=1e-12)
        elif r["units"] == "frame-of-reference":
            assert r["raw_share_k"] < 1.0 and r["raw_share_v"] < 1.0
            assert r["cr_k"] > r["plain_quant_cr"] and r["cr_v"] > r["plain_quant_cr"]
        if r["units"] == "width-only":
            f = by[(r["inputs"], r["bits"], r["reorder_key"], "frame-of-reference")]
            assert r["cr_k"] <= f["cr_k"] and r["cr_v"] <= f["cr_v"]
