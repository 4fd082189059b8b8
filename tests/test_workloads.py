"""The synthetic inputs follow their stated recipe: shapes and settings of each
workload, draft = target + Gaussian noise of the stated sigma, the greedy
workload's tied rows, the mixed temperatures, the +12 spikes, and counter-based
generation (a row does not depend on the batch size; a seed fixes every byte)."""
import numpy as np
import pytest

import workloads


def _f(a, dtype):
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if dtype == "bf16" else a.astype(np.float64)


@pytest.mark.parametrize("name,B,k,V,dtype,mode,top_k", [
    ("tiny", 1, 4, 32, "f32", "stochastic", 0),
    ("single", 1, 8, 151936, "bf16", "stochastic", 0),
    ("batched", 64, 4, 151936, "bf16", "stochastic", 50),
    ("greedy", 256, 8, 151936, "bf16", "greedy", 0),
    ("large", 512, 3, 128256, "f32", "stochastic", 0),
])
def test_workload_settings(name, B, k, V, dtype, mode, top_k):
    w = workloads.WORKLOADS[name]
    assert (w.B, w.k, w.V, w.dtype, w.mode, w.top_k) == (B, k, V, dtype, mode, top_k)
    rows = (k + 1) if mode == "greedy" else (2 * k + 1)
    assert workloads.workload_bytes(B, k, V, 2 if dtype == "bf16" else 4, mode) == B * rows * V * (2 if dtype == "bf16" else 4)


@pytest.mark.parametrize("name", ["tiny", "batched", "large"])
def test_draft_is_target_plus_noise_of_the_stated_sigma(name):
    w = workloads.WORKLOADS[name]
    case = workloads.make_case(name, seed=5, B=2, V=min(w.V, 20000))
    t = _f(case.target[:, :case.k], case.dtype)
    d = _f(case.draft, case.dtype)
    noise = (d - t).ravel()
    tol = 0.05 * w.draft_sigma + (0.02 if case.dtype == "bf16" else 0.0)
    if noise.size > 1000:
        assert abs(noise.mean()) < tol
        assert abs(noise.std() - w.draft_sigma) < tol
    # the target itself: N(0, sigma^2) away from the spikes
    tt = _f(case.target, case.dtype).ravel()
    if tt.size > 1000:
        core = tt[np.abs(tt) < 8 * w.target_sigma]
        assert abs(core.std() - w.target_sigma) < 0.05 * w.target_sigma


def test_spikes_raise_five_entries_per_target_row(monkeypatch):
    """Against the same seed generated without spikes, exactly five entries of
    every target row differ, each by +12 (up to bf16 rounding), and the draft
    rows carry the same spikes (the draft is built from the spiked target)."""
    import dataclasses

    spiked = workloads.make_case("batched", seed=9, B=2, V=4096)
    plain_w = dataclasses.replace(workloads.WORKLOADS["batched"], spikes=0)
    monkeypatch.setitem(workloads.WORKLOADS, "batched", plain_w)
    plain = workloads.make_case("batched", seed=9, B=2, V=4096)
    d = (_f(spiked.target, "bf16") - _f(plain.target, "bf16")).reshape(-1, 4096)
    for row in d:
        moved = np.nonzero(np.abs(row) > 1.0)[0]
        assert moved.size == 5
        assert np.all(np.abs(row[moved] - workloads.SPIKE) < 0.25)
    dd = (_f(spiked.draft, "bf16") - _f(plain.draft, "bf16")).reshape(-1, 4096)
    assert all(np.sum(np.abs(r) > 1.0) == 5 for r in dd)


def test_greedy_tie_rows():
    """About 1 % of the target rows hold their maximum, the planted value 30, at
    exactly two indices (N(0, 9) entries never come near 30)."""
    case = workloads.make_case("greedy", seed=3, B=256, V=2048)
    t = _f(case.target, "bf16").reshape(-1, 2048)
    planted = t.max(axis=1) == workloads.TIE_VALUE
    assert 0.002 < planted.mean() < 0.03
    assert np.all(np.sum(t[planted] == workloads.TIE_VALUE, axis=1) == 2)
    assert case.draft is None and case.draft_proxy is not None


def test_large_workload_mixes_three_temperatures():
    case = workloads.make_case("large", seed=2, B=300, V=64)
    vals, counts = np.unique(case.temperature, return_counts=True)
    assert vals.tolist() == [0.5, 1.0, 1.5]
    assert counts.min() > 60


def test_rows_do_not_depend_on_the_batch_size():
    a = workloads.make_case("batched", seed=4, B=2, V=3000)
    b = workloads.make_case("batched", seed=4, B=5, V=3000)
    assert np.array_equal(a.target, b.target[:2])
    assert np.array_equal(a.uniforms, b.uniforms[:2])
    c = workloads.make_case("batched", seed=5, B=2, V=3000)
    assert not np.array_equal(a.target, c.target)


def test_uniforms_and_dtypes():
    case = workloads.make_case("batched", seed=1, B=3, V=1000)
    assert case.target.dtype == np.uint16 and case.draft.dtype == np.uint16
    assert case.uniforms.shape == (3, 5) and case.draft_uniforms.shape == (3, 4)
    for u in (case.uniforms, case.draft_uniforms):
        assert u.dtype == np.float32 and np.all(u >= 0) and np.all(u < 1)
    assert np.all(case.temperature == np.float32(0.7))
