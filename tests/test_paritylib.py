"""The parity checker rejects what it must: results built from the oracle's
own output pass, and each planted discrepancy (a wrong token, count, p or q
beyond 1e-5, a missed row error, a broken prefix at a flagged decision, a
final token outside its CDF window) makes it fail.  CPU only."""
import copy

import numpy as np
import pytest

import oracle
from paritylib import (DECISION_TOL, GpuResult, compare, compare_samples, flag_probability,
                       nucleus_near_cut)


def _case(seed=0, B=12, k=3, V=40, top_k=0):
    rng = np.random.default_rng(seed)
    target = rng.normal(0, 2, (B, k + 1, V)).astype(np.float32)
    draft = (target[:, :k] + rng.normal(0, 1, (B, k, V))).astype(np.float32)
    temp = rng.uniform(0.6, 1.4, B).astype(np.float32)
    u = rng.uniform(0, 1, (B, k + 1)).astype(np.float32)
    drafts = oracle.sample_rows(draft, u[:, :k], np.repeat(temp, k), top_k)[0].astype(np.int32)
    ref = oracle.verify(target, draft, drafts, u, temp, top_k)
    return target, draft, drafts, u, temp, top_k, ref


def _as_gpu(ref):
    return GpuResult(ref.tokens.copy(), ref.n_accepted.copy(), ref.p.astype(np.float32),
                     ref.q.astype(np.float32), 0)


def _inputs(c):
    target, draft, drafts, u, temp, top_k, _ = c
    return (target, draft, drafts, temp, top_k)


def test_oracle_output_passes():
    c = _case()
    ref = c[-1]
    rep = compare(ref, _as_gpu(ref), c[3], inputs=_inputs(c))
    assert rep.exact + rep.flagged == rep.sequences and rep.errors == 0
    assert rep.max_p_err < 1e-7 and rep.max_q_err < 1e-7


def _first(ref, pred):
    for b in range(ref.tokens.shape[0]):
        if pred(b):
            return b
    pytest.skip("the seeded case has no sequence of this kind")


@pytest.mark.parametrize("fault", ["token", "count", "p", "q", "tail"])
def test_planted_discrepancies_fail(fault):
    c = _case(1)
    ref = c[-1]
    gpu = _as_gpu(ref)
    b = _first(ref, lambda b: 0 <= ref.n_accepted[b] < ref.tokens.shape[1] - 1)
    j = int(ref.n_accepted[b])
    if fault == "token":
        gpu.tokens[b, j] = (gpu.tokens[b, j] + 1) % c[0].shape[-1]
    elif fault == "count":
        gpu.n_accepted[b] += 1
    elif fault == "p":
        gpu.p[b, 0] += 2 * DECISION_TOL
    elif fault == "q":
        gpu.q[b, 0] -= 2 * DECISION_TOL
    else:
        gpu.tokens[b, j + 1] = 0
    with pytest.raises(AssertionError):
        compare(ref, gpu, c[3], inputs=_inputs(c))


def test_missed_row_error_fails():
    c = list(_case(2))
    target = c[0].copy()
    target[3, 1, 5] = np.nan
    c[0] = target
    ref = oracle.verify(target, c[1], c[2], c[3], c[4], c[5])
    assert ref.n_accepted[3] == -1
    good = _as_gpu(ref)
    compare(ref, good, c[3])
    bad = copy.deepcopy(good)
    bad.n_accepted[3] = 0
    with pytest.raises(AssertionError):
        compare(ref, bad, c[3])
    bad = copy.deepcopy(good)
    bad.tokens[3, 0] = 7
    with pytest.raises(AssertionError):
        compare(ref, bad, c[3])


def test_flagged_acceptance_keeps_the_prefix_check():
    """A uniform set on an acceptance threshold is counted; the tokens before
    that position must still match, the rest may differ."""
    c = list(_case(3, B=16))
    ref = c[-1]
    b = _first(ref, lambda b: ref.n_accepted[b] >= 2)
    u = c[3].copy()
    u[b, 1] = np.float32(ref.ratio[b, 1])      # on the threshold of position 1
    ref = oracle.verify(c[0], c[1], c[2], u, c[4], c[5])
    gpu = _as_gpu(ref)
    gpu.n_accepted[b] = 1
    gpu.tokens[b, 1:] = -1
    gpu.tokens[b, 1] = 0                       # a different decision past the flag is allowed
    rep = compare(ref, gpu, u, inputs=(c[0], c[1], c[2], c[4], c[5]))
    assert rep.flagged_accept >= 1
    gpu.tokens[b, 0] = (ref.tokens[b, 0] + 1) % c[0].shape[-1]   # the prefix is not
    with pytest.raises(AssertionError):
        compare(ref, gpu, u, inputs=(c[0], c[1], c[2], c[4], c[5]))


def test_flagged_final_draw_checks_the_window():
    """A final uniform on a CDF point is counted; the token on the other side
    of that point is accepted, a token whose interval is far from u_k is not."""
    c = list(_case(4, B=16))
    ref = c[-1]
    b = _first(ref, lambda b: ref.n_accepted[b] >= 0 and 0.05 < ref.cdf_lo[b] < 0.95)
    k = ref.tokens.shape[1] - 1
    u = c[3].copy()
    u[b, k] = np.float32(ref.cdf_lo[b])
    ref = oracle.verify(c[0], c[1], c[2], u, c[4], c[5])
    j = int(ref.n_accepted[b])
    ins = (c[0], c[1], c[2], c[4], c[5])
    gpu = _as_gpu(ref)
    rep = compare(ref, gpu, u, inputs=ins)
    assert rep.flagged_final >= 1
    y = int(ref.tokens[b, j])
    pos = np.nonzero(_weights(c, b, j, ref))[0]
    at_lo = abs(float(u[b, k]) - ref.cdf_lo[b]) < DECISION_TOL
    other = pos[pos < y].max() if at_lo else pos[pos > y].min()
    gpu.tokens[b, j] = other                   # across the flagged CDF point: allowed
    compare(ref, gpu, u, inputs=ins)
    C = np.cumsum(_weights(c, b, j, ref))
    C /= C[-1]
    far = [v for v in pos if min(abs(C[v] - u[b, k]), abs((C[v - 1] if v else 0.0) - u[b, k])) > 0.05
           and not ((C[v - 1] if v else 0.0) <= u[b, k] <= C[v])]
    assert far
    gpu.tokens[b, j] = far[0]
    with pytest.raises(AssertionError):
        compare(ref, gpu, u, inputs=ins)


def _weights(c, b, j, ref):
    T = float(c[4][b])
    pt = oracle.process_row(c[0][b, j], T, c[5])
    if j < ref.tokens.shape[1] - 1:
        r = np.maximum(0.0, pt - oracle.process_row(c[1][b, j], T, c[5]))
        if r.sum() > 0:
            return r
    return pt


def test_greedy_is_bit_exact():
    rng = np.random.default_rng(5)
    target = rng.normal(0, 1, (6, 3, 30)).astype(np.float32)
    drafts = rng.integers(0, 30, (6, 2)).astype(np.int32)
    drafts[0] = [int(np.argmax(target[0, 0])), int(np.argmax(target[0, 1]))]
    ref = oracle.verify(target, None, drafts, None, greedy=True)
    gpu = GpuResult(ref.tokens.copy(), ref.n_accepted.copy(), ref.p, ref.q, 0)
    compare(ref, gpu, None, greedy=True)
    gpu.tokens[0, 2] = (gpu.tokens[0, 2] + 1) % 30
    with pytest.raises(AssertionError):
        compare(ref, gpu, None, greedy=True)


@pytest.mark.parametrize("probs,top_p,near", [
    ([0.5, 0.3, 0.2], 0.8, True),             # the running sum hits top_p exactly at a step
    ([0.5, 0.3, 0.2], 0.799995, True),        # within 1e-5 below that step
    ([0.5, 0.3, 0.2], 0.7, False),
    ([0.5, 0.3, 0.2], 0.500005, True),        # just past the previous step
    ([0.6, 0.4], 1.0, False),                 # no nucleus
    ([0.25, 0.25, 0.25, 0.25], 0.6, False),
])
def test_nucleus_near_cut_hand_cases(probs, top_p, near):
    assert bool(nucleus_near_cut(np.array(probs), top_p)) == near


# ---- the proposer-sampler comparison ------------------------------------------------

def _sample_case(seed=3, rows=60, V=400, top_k=0):
    rng = np.random.default_rng(seed)
    logits = rng.normal(0, 2, (rows, V)).astype(np.float32)
    temp = np.asarray([0.5, 1.0, 1.5], np.float32)[np.arange(rows) % 3]
    u = rng.uniform(0, 1, rows).astype(np.float32)
    ref, lo, hi = oracle.sample_rows(logits, u, temp, top_k)
    return logits, u, temp, top_k, ref, lo, hi


def test_flag_probability_matches_a_fine_grid():
    """The flagged measure of [0, 1) under the rule, counted on a grid of u."""
    w = np.array([0.5, 1e-6, 0.0, 3e-6, 0.25, 0.25 - 4e-6])
    G = 2_000_000
    u = (np.arange(G) + 0.5) / G
    C = np.cumsum(w) / w.sum()
    tok = np.searchsorted(C, u, side="right")
    lo = np.where(tok > 0, C[np.maximum(tok - 1, 0)], 0.0)
    hi = C[tok]
    flagged = (np.abs(u - lo) < DECISION_TOL) | (np.abs(u - hi) < DECISION_TOL)
    assert abs(flagged.mean() - flag_probability(w)) < 2.0 / G * 8


def test_sampler_oracle_output_passes_and_counts():
    logits, u, temp, top_k, ref, lo, hi = _sample_case()
    rep = compare_samples(logits, u, temp, top_k, ref.copy(), ref, lo, hi)
    assert rep.exact + rep.flagged == rep.rows


def test_sampler_wrong_token_fails():
    logits, u, temp, top_k, ref, lo, hi = _sample_case()
    near = (np.abs(u - lo) < DECISION_TOL) | (np.abs(u - hi) < DECISION_TOL)
    r = int(np.flatnonzero(~near)[0])
    got = ref.copy()
    got[r] = (got[r] + 1) % logits.shape[1]
    with pytest.raises(AssertionError):
        compare_samples(logits, u, temp, top_k, got, ref, lo, hi)


def test_sampler_flagged_row_checks_the_window():
    """A flagged row whose GPU token lies far from u in the CDF fails."""
    logits, u, temp, top_k, ref, lo, hi = _sample_case(rows=3)
    u = u.copy()
    u[0] = np.float32(hi[0])  # on the CDF point above the oracle's token: flagged
    ref2, lo2, hi2 = oracle.sample_rows(logits, u, temp, top_k)
    got = ref2.copy()
    w = oracle.process_row(logits[0], float(temp[0]), top_k)
    C = np.cumsum(w) / w.sum()
    far = int(np.argmax(np.abs(C - u[0]) > 0.1))
    got[0] = far
    with pytest.raises(AssertionError):
        compare_samples(logits, u, temp, top_k, got, ref2, lo2, hi2)
    got[0] = ref2[0]
    assert compare_samples(logits, u, temp, top_k, got, ref2, lo2, hi2).flagged >= 1


def test_sampler_flag_count_is_bounded():
    """More flagged rows than the rule predicts fails: uniforms planted on CDF points."""
    logits, u, temp, top_k, ref, lo, hi = _sample_case(rows=40)
    u = hi.astype(np.float32)  # every row on a CDF point
    ref2, lo2, hi2 = oracle.sample_rows(logits, u, temp, top_k)
    with pytest.raises(AssertionError):
        compare_samples(logits, u, temp, top_k, ref2.copy(), ref2, lo2, hi2)
