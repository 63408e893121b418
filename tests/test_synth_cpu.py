"""The seeded input generators (no method arithmetic): reproducible, identical whether a
sequence is drawn at once or from an offset, and with the shapes and statistics the
workload recipe states."""
import numpy as np
import pytest

from decode_gemv_packkv_b200 import synth


@pytest.mark.parametrize("structured", [False, True])
def test_slices_are_reproducible_and_offset_consistent(structured):
    k0, v0 = synth.kv_slice(1234, 4, 1, 2, 700, structured=structured)
    k1, v1 = synth.kv_slice(1234, 4, 1, 2, 700, structured=structured)
    assert k0.dtype == np.float16 and k0.shape == (700, 128) and v0.shape == (700, 128)
    assert np.array_equal(k0, k1) and np.array_equal(v0, v1)
    k2, v2 = synth.kv_slice(1234, 4, 1, 2, 300, start=400, structured=structured)
    assert np.array_equal(k2, k0[400:]) and np.array_equal(v2, v0[400:])
    k3, _ = synth.kv_slice(1234, 4, 1, 3, 700, structured=structured)  # another head differs
    assert not np.array_equal(k3, k0)


def test_iid_statistics_follow_the_recipe():
    """K[t, c] = mu_c + sigma_c N(0, 1) with sigma_c in [0.5, 2] except 4 outlier channels
    at 10x; V ~ N(0, 1)."""
    k, v = synth.kv_slice(99, 1, 0, 0, 8192)
    sd = k.astype(np.float64).std(axis=0)
    outliers = np.sort(sd)[-4:]
    assert np.all(outliers > 4.0)                      # 10 x sigma >= 5
    assert np.all(np.sort(sd)[:-4] < 2.2) and np.all(np.sort(sd)[:-4] > 0.4)
    assert abs(v.astype(np.float64).mean()) < 0.01 and abs(v.astype(np.float64).std() - 1) < 0.01


def test_structured_inputs_hold_few_levels_for_runs():
    """Every channel takes at most 16 distinct values and repeats its previous value
    inside its run; the first token of each run may change it."""
    k, v = synth.kv_slice(5, 1, 0, 0, 1000, structured=True)
    for x in (k, v):
        for c in range(128):
            assert len(np.unique(x[:, c])) <= 16
        same = (x[1:] == x[:-1]).mean()
        assert same > 0.5                              # runs of 1..47 tokens


def test_queries_and_timing_probabilities():
    w = synth.WORKLOADS[2]
    q0, q1 = synth.queries(w, 0), synth.queries(w, 1)
    assert q0.shape == (w.batch, w.q_heads, 128) and q0.dtype == np.float16
    assert not np.array_equal(q0, q1)
    p = synth.timing_probs(w, 1000)
    assert p.shape == (w.batch, w.q_heads, 1000) and np.all(p >= 0)
    assert np.allclose(p.sum(axis=-1), 1.0, atol=1e-5)
