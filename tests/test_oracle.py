"""Pins of the fp64 oracle against facts that do not come from the oracle.

* the pages' worked example (golden fixture ``tests/golden/worked_example.json``);
* distribution preservation, checked EXACTLY by brute force at V <= 4, k <= 2:
  the sampler's output is piecewise constant in each uniform, so evaluating
  it at the midpoint of every constant piece and weighting by piece length
  gives the exact output law, which must reproduce the target at every
  position (speculative decoding entry "推测解码", section
  "提议与核验的基本步骤", paragraphs 2-3: accepted drafts plus corrections
  keep the target distribution);
* a chi-square test of the emitted tokens on the tiny workload;
* closed forms of the softmax (uniform rows, the logistic two-token case);
* hand cases of top-k with ties, of the lowest-index argmax and of the
  inverse CDF;
* the published splitmix64 reference outputs and bf16 round-to-nearest-even.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy import stats

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# generator pins
# --------------------------------------------------------------------------

def test_splitmix64_reference_outputs():
    # first five outputs of the reference splitmix64 seeded with 1234567
    expected = [6457827717110365317, 3203168211198807973, 9817491932198370423,
                4593380528125082431, 16408922859458223821]
    assert [int(x) for x in workloads.splitmix64_stream(1234567, 5)] == expected


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, -0.0, 3e38])
    bits = workloads.f64_to_bf16_bits(x)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000, 0x8000, 0x7F62]
    assert workloads.bf16_bits_to_f32(np.array([0x3F80, 0xC020], np.uint16)).tolist() == [1.0, -2.5]


def test_uniforms_are_in_unit_interval_and_24_bit():
    u = workloads.uniform_f32(7, workloads.TAG_UNIFORMS, 64, 33)
    assert u.dtype == np.float32 and u.min() >= 0.0 and u.max() < 1.0
    assert np.all((u.astype(np.float64) * 2 ** 24) == np.floor(u.astype(np.float64) * 2 ** 24))


def test_normals_moments():
    z = workloads.normals_f64(3, workloads.TAG_TARGET, np.arange(8), 50000).ravel()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


# --------------------------------------------------------------------------
# softmax / processing closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("V", [1, 7, 32])
def test_equal_logits_give_uniform(V):
    prob = oracle.process_row(np.full(V, 1.5, np.float32))
    assert np.allclose(prob, 1.0 / V, rtol=0, atol=1e-15)


@pytest.mark.parametrize("delta,T", [(0.0, 1.0), (1.0, 1.0), (2.5, 0.7), (-3.0, 1.5), (12.0, 0.5)])
def test_two_token_logistic(delta, T):
    prob = oracle.process_row(np.array([0.0, delta], np.float32), temperature=T)
    expect = 1.0 / (1.0 + math.exp(-float(np.float32(delta)) / T))
    assert abs(prob[1] - expect) < 1e-15 and abs(prob.sum() - 1.0) < 1e-15


def test_bf16_row_uses_widened_values():
    bits = workloads.f64_to_bf16_bits(np.array([0.0, 1.0, 2.0]))
    prob = oracle.process_row(bits)
    e = np.exp([0.0, 1.0, 2.0])
    assert np.allclose(prob, e / e.sum(), rtol=0, atol=1e-15)


def test_neg_inf_entries_get_zero_mass():
    prob = oracle.process_row(np.array([0.0, -np.inf, 0.0, -np.inf], np.float32))
    assert prob.tolist() == [0.5, 0.0, 0.5, 0.0]


@pytest.mark.parametrize("row,K,kept", [
    ([3, 3, 2, 1], 1, [0, 1]),            # tie at the threshold: both kept
    ([3, 3, 2, 1], 2, [0, 1]),
    ([3, 3, 2, 1], 3, [0, 1, 2]),
    ([5, 4, 4, 4, 1], 2, [0, 1, 2, 3]),   # tau = 4 straddles three entries
    ([2, 2, 2, 2], 2, [0, 1, 2, 3]),      # all equal: everything kept
    ([1, -0.0, 0.0, -1], 2, [0, 1, 2]),   # -0 and +0 are the same value
    ([1, 4, 2, 3], 4, [0, 1, 2, 3]),      # K = V disables top-k
    ([1, 4, 2, 3], 9, [0, 1, 2, 3]),      # K > V disables top-k
    ([1, 4, 2, 3], 0, [0, 1, 2, 3]),      # K = 0 disables top-k
])
def test_top_k_hand_cases(row, K, kept):
    z = np.array(row, np.float32)
    prob = oracle.process_row(z, top_k=K)
    assert np.nonzero(prob > 0)[0].tolist() == kept
    e = np.exp(z[kept].astype(np.float64) - z[kept].max())
    assert np.allclose(prob[kept], e / e.sum(), rtol=0, atol=1e-15)


@pytest.mark.parametrize("seed", range(6))
def test_top_k_invariants_random_rows(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(5, 300))
    z = np.round(rng.normal(0, 2, V) * 2) / 2          # coarse grid: many ties
    bits = workloads.f64_to_bf16_bits(z)
    zz = workloads.bf16_bits_to_f32(bits).astype(np.float64)
    for K in (1, 2, 5, V // 2, V - 1):
        prob = oracle.process_row(bits, temperature=0.8, top_k=K)
        kept = prob > 0
        assert kept.sum() >= K
        assert zz[kept].min() >= zz[~kept].max() if (~kept).any() else True
        assert (zz > zz[kept].min()).sum() < K


def test_temperature_scales_logits():
    p1 = oracle.process_row(np.array([0.0, 1.0], np.float32), temperature=0.5)
    p2 = oracle.process_row(np.array([0.0, 2.0], np.float32), temperature=1.0)
    assert np.allclose(p1, p2, rtol=0, atol=1e-15)


@pytest.mark.parametrize("row", [[0.0, np.nan, 1.0], [0.0, np.inf], [-np.inf, -np.inf]])
def test_bad_rows_are_errors(row):
    assert oracle.process_row(np.array(row, np.float32)) is None


@pytest.mark.parametrize("T", [0.0, -1.0, np.inf, np.nan])
def test_bad_temperature_is_error(T):
    assert oracle.process_row(np.array([0.0, 1.0], np.float32), temperature=T) is None


# --------------------------------------------------------------------------
# greedy
# --------------------------------------------------------------------------

@pytest.mark.parametrize("row,expect", [
    ([1, 5, 5, 2], 1),
    ([-0.0, 0.0, -1.0], 0),
    ([0.0, -0.0, -1.0], 0),
    ([-np.inf, -np.inf, 3, 3], 2),
    ([7], 0),
    ([-np.inf, -np.inf], -1),
    ([1, np.nan], -1),
    ([1, np.inf], -1),
])
def test_argmax_lowest_index(row, expect):
    assert oracle.argmax_row(np.array(row, np.float32)) == expect


def test_greedy_verify_rule():
    target = np.array([[[1, 5, 5, 2], [0, 0, 9, 9], [-0.0, 0.0, -1, -2]]], np.float32)
    # argmaxes 1, 2, 0; the first mismatch decides, a later one changes nothing
    cases = [([1, 2], 2, [1, 2, 0]), ([2, 2], 0, [1, -1, -1]), ([1, 3], 1, [1, 2, -1]),
             ([2, 3], 0, [1, -1, -1])]
    for d, n, toks in cases:
        r = oracle.verify(target, None, np.array([d]), None, greedy=True)
        assert r.n_accepted.tolist() == [n] and r.tokens[0].tolist() == toks


# --------------------------------------------------------------------------
# inverse CDF
# --------------------------------------------------------------------------

@pytest.mark.parametrize("w,u,expect,lo_hi", [
    ([0, 1, 0, 3], 0.0, 1, (0.0, 0.25)),           # zero-weight entries are never drawn
    ([0, 1, 0, 3], 0.2499, 1, (0.0, 0.25)),
    ([0, 1, 0, 3], 0.25, 3, (0.25, 1.0)),          # C_v > u*W is strict
    ([0, 1, 0, 3], 0.999, 3, (0.25, 1.0)),
    ([1, 2, 0], 1.0 - 2 ** -53, 1, (1 / 3, 1.0)),  # u just below 1: the last positive entry
    ([5], 0.5, 0, (0.0, 1.0)),
    ([2, 1, 1], 0.6, 1, (0.5, 0.75)),
])
def test_inverse_cdf_hand_cases(w, u, expect, lo_hi):
    """Token and the CDF points C_{y-1}/W, C_y/W around it (reading R3)."""
    tok, lo, hi = oracle.inverse_cdf(np.array(w, np.float64), u)
    assert tok == expect
    assert lo == pytest.approx(lo_hi[0], abs=1e-15) and hi == pytest.approx(lo_hi[1], abs=1e-15)


def test_inverse_cdf_zero_mass():
    assert oracle.inverse_cdf(np.zeros(4), 0.3) is None


# --------------------------------------------------------------------------
# the pages' worked example
# --------------------------------------------------------------------------

def _worked_example():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        g = json.load(f)
    p = np.array(g["target_probs"])
    q = np.array(g["draft_probs"])
    target = np.log(np.stack([p, p])).astype(np.float32)[None]    # position 0 and bonus row
    draft = np.log(q).astype(np.float32)[None, None]
    return g, target, draft


def test_worked_example_acceptance_and_residual():
    g, target, draft = _worked_example()
    d = np.array([[g["draft_token"]]])
    r = oracle.verify(target, draft, d, np.array([[0.5, 0.5]], np.float32))
    assert abs(r.q[0, 0] - g["draft_token_probability"]) < 1e-6
    assert abs(r.ratio[0, 0] - g["accept_probability"]) < 1e-6
    # u just below the ratio accepts (then the bonus row is sampled), just above rejects
    acc = oracle.verify(target, draft, d, np.array([[0.7499, 0.5]], np.float32))
    assert acc.n_accepted[0] == 1 and acc.tokens[0, 0] == g["draft_token"]
    # u exactly at 0.75 sits inside the 1e-5 near-threshold window
    assert abs(0.75 - r.ratio[0, 0]) < 1e-5
    # on rejection the residual max(0, p - q) lives on A only, for any final uniform
    uk = np.linspace(0.0, 0.999, 101, dtype=np.float32)
    B = uk.size
    rej = oracle.verify(np.repeat(target, B, 0), np.repeat(draft, B, 0), np.repeat(d, B, 0),
                        np.stack([np.full(B, 0.7501, np.float32), uk], 1))
    assert np.all(rej.n_accepted == 0)
    assert set(rej.tokens[:, 0].tolist()) == set(g["residual_support"])


def test_worked_example_recombined_marginals():
    g, target, draft = _worked_example()
    G = 4096
    mid = ((np.arange(G) + 0.5) / G).astype(np.float32)
    marg = np.zeros(3)
    for dtok, qd in enumerate(g["draft_probs"]):
        d = np.full((G, 1), dtok)
        # acceptance fraction over the first uniform (final uniform fixed)
        r = oracle.verify(np.repeat(target, G, 0), np.repeat(draft, G, 0), d,
                          np.stack([mid, np.full(G, 0.5, np.float32)], 1))
        acc = np.mean(r.n_accepted == 1)
        # replacement law over the final uniform, first uniform forcing rejection
        r2 = oracle.verify(np.repeat(target, G, 0), np.repeat(draft, G, 0), d,
                           np.stack([np.full(G, 0.9999999, np.float32), mid], 1))
        rejected = r2.n_accepted == 0
        res = np.bincount(r2.tokens[rejected, 0], minlength=3) / max(1, rejected.sum())
        marg[dtok] += qd * acc
        marg += qd * (1 - acc) * res
    assert np.allclose(marg, g["recombined_marginals"], rtol=0, atol=1e-6)


# --------------------------------------------------------------------------
# exact brute force of the output law (V <= 4, k <= 2)
# --------------------------------------------------------------------------

def _pieces(points):
    pts = sorted(set([0.0, 1.0] + [float(x) for x in points if 0.0 < x < 1.0]))
    return [(a, b) for a, b in zip(pts[:-1], pts[1:]) if b - a > 1e-6]


def _exact_law(target, draft, T, top_k):
    """Exact joint law of (n, emitted tokens) of the oracle's sampler."""
    k, V = draft.shape
    p = [oracle.process_row(target[i], T, top_k) for i in range(k + 1)]
    q = [oracle.process_row(draft[i], T, top_k) for i in range(k)]
    # every CDF point the final uniform may be compared against
    fpts = []
    for j in range(k):
        for w in (np.maximum(0.0, p[j] - q[j]), p[j]):
            if w.sum() > 0:
                fpts += list(np.cumsum(w) / w.sum())
    fpts += list(np.cumsum(p[k]) / p[k].sum())
    fin = _pieces(fpts)
    rows, weights = [], []
    for d in itertools.product(range(V), repeat=k):
        wd = np.prod([q[i][d[i]] for i in range(k)])
        if wd == 0:
            continue
        slots = []
        for i in range(k):
            r = min(1.0, p[i][d[i]] / q[i][d[i]])
            slots.append(_pieces([r]))
        for acc in itertools.product(*slots):
            for f in fin:
                u = [0.5 * (a + b) for a, b in acc] + [0.5 * (f[0] + f[1])]
                wt = wd * np.prod([b - a for a, b in acc]) * (f[1] - f[0])
                rows.append((d, u))
                weights.append(wt)
    B = len(rows)
    tk = np.array([r[0] for r in rows], np.int32).reshape(B, k)
    uu = np.array([r[1] for r in rows], np.float32)
    res = oracle.verify(np.repeat(target[None], B, 0), np.repeat(draft[None], B, 0), tk, uu,
                        np.full(B, T, np.float32), top_k)
    dropped = 1.0 - float(np.sum(weights))
    return p, q, res, np.array(weights), dropped


@pytest.mark.parametrize("V,k", [(2, 1), (3, 1), (3, 2), (4, 1), (4, 2)])
@pytest.mark.parametrize("T,top_k", [(1.0, 0), (0.6, 0), (1.3, 2)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_distribution_preservation(V, k, T, top_k, seed):
    rng = np.random.default_rng(1000 * V + 100 * k + seed)
    target = rng.normal(0, 1.5, (k + 1, V)).astype(np.float32)
    draft = (target[:k] + rng.normal(0, 1.0, (k, V))).astype(np.float32)
    p, q, res, wts, dropped = _exact_law(target, draft, T, top_k)
    assert res.errors == 0
    tol = 1e-9 + abs(dropped)
    n = res.n_accepted
    for m in range(k + 1):
        reach = n >= m
        P_reach = wts[reach].sum()
        law = np.array([wts[reach & (res.tokens[:, m] == v)].sum() for v in range(V)])
        assert np.allclose(law / P_reach, p[m], rtol=0, atol=tol / max(P_reach, 1e-300)), (m, law / P_reach, p[m])
        if m < k:
            # acceptance rate identity: P(accept at m | reached m) = sum_v min(p_m, q_m)
            P_next = wts[n >= m + 1].sum()
            assert abs(P_next / P_reach - np.minimum(p[m], q[m]).sum()) < tol / P_reach


# --------------------------------------------------------------------------
# chi-square on the tiny workload
# --------------------------------------------------------------------------

def test_chi_square_emitted_law():
    case = workloads.make_case("tiny", seed=11)
    k, V = case.k, case.V
    p = [oracle.process_row(case.target[0, i]) for i in range(k + 1)]
    q0 = oracle.process_row(case.draft[0, 0])
    counts = np.zeros((k + 1, V))
    reached = np.zeros(k + 1)
    n_total = 0
    for rep in range(10):
        B = 100_000
        du = workloads.uniform_f32(500 + rep, workloads.TAG_DRAFT_UNIFORMS, B, k)
        uu = workloads.uniform_f32(500 + rep, workloads.TAG_UNIFORMS, B, k + 1)
        drafts = np.ascontiguousarray(np.broadcast_to(case.draft, (B, k, V)))
        dtok, _, _ = oracle.sample_rows(drafts, du)
        r = oracle.verify(np.ascontiguousarray(np.broadcast_to(case.target, (B, k + 1, V))), drafts,
                          dtok, uu)
        for m in range(k + 1):
            sel = r.n_accepted >= m
            reached[m] += sel.sum()
            counts[m] += np.bincount(r.tokens[sel, m], minlength=V)
        n_total += B
    for m in range(k + 1):
        exp = reached[m] * p[m]
        big = exp >= 5
        obs = np.append(counts[m][big], counts[m][~big].sum())
        ex = np.append(exp[big], exp[~big].sum())
        if ex[-1] == 0:
            obs, ex = obs[:-1], ex[:-1]
        assert stats.chisquare(obs, ex).pvalue > 1e-3, m
    # acceptance at position 0 matches sum_v min(p_0, q_0)
    a = reached[1] / n_total
    alpha = np.minimum(p[0], q0).sum()
    assert abs(a - alpha) < 5 * math.sqrt(alpha * (1 - alpha) / n_total)


@pytest.mark.parametrize("u,expect", [(0.0, 0), (0.1, 0), (0.25, 1), (0.3, 1), (0.5, 2), (0.9, 3)])
def test_sampler_token_for_each_uniform(u, expect):
    """Four equal logits give 1/4 each, so the draw is the smallest v with
    (v + 1)/4 > u (reading R3): the map from u to the token is fixed, not only
    its law."""
    row = np.zeros((1, 4), np.float32)
    tok, lo, hi = oracle.sample_rows(row, np.array([u], np.float32), np.ones(1, np.float32))
    assert tok[0] == expect and lo[0] == expect / 4 and hi[0] == (expect + 1) / 4


def test_sampler_law_by_midpoint_grid():
    """The proposer/bonus draw of a row reproduces its processed distribution."""
    row = np.array([0.3, -1.0, 2.0, 0.0, 1.1], np.float32)
    prob = oracle.process_row(row, temperature=0.9)
    G = 1 << 16
    mid = ((np.arange(G) + 0.5) / G).astype(np.float32)
    tok, _, _ = oracle.sample_rows(np.repeat(row[None], G, 0), mid, np.full(G, 0.9, np.float32))
    assert np.allclose(np.bincount(tok, minlength=5) / G, prob, rtol=0, atol=2.0 / G)


# --------------------------------------------------------------------------
# special cases and error semantics
# --------------------------------------------------------------------------

def test_draft_outside_draft_top_k_is_accepted_when_target_keeps_it():
    target = np.array([[[0, 0, 0, 0], [0, 0, 0, 0]]], np.float32)       # p uniform
    draft = np.array([[[5, 0, 0, 0]]], np.float32)                      # q top-1: only id 0
    r = oracle.verify(target, draft, np.array([[2]]), np.array([[0.99, 0.1]], np.float32), top_k=1)
    # q(2) = 0 < p(2)?  p with top-1 keeps all four tied entries
    assert r.q[0, 0] == 0.0 and r.p[0, 0] == 0.25 and r.n_accepted[0] == 1


def test_zero_residual_mass_falls_back_to_target():
    row = np.array([0, 3, 1, 2], np.float32)
    target = np.stack([row, row])[None]
    draft = row[None, None]
    # top-1 on both sides: p = q = one-hot at id 1; the draft token 0 has p = q = 0
    r = oracle.verify(target, draft, np.array([[0]]), np.array([[0.2, 0.6]], np.float32), top_k=1)
    assert r.n_accepted[0] == 0 and r.tokens[0, 0] == 1


@pytest.mark.parametrize("what", ["token_low", "token_high", "temp_zero", "temp_nan", "u_one",
                                  "u_neg", "nan_logit", "inf_logit", "all_neg_inf"])
def test_row_errors(what):
    V, k = 5, 2
    target = np.zeros((2, k + 1, V), np.float32)
    draft = np.zeros((2, k, V), np.float32)
    d = np.ones((2, k), np.int32)
    u = np.full((2, k + 1), 0.5, np.float32)
    T = np.ones(2, np.float32)
    if what == "token_low": d[0, 1] = -1
    if what == "token_high": d[0, 0] = V
    if what == "temp_zero": T[0] = 0.0
    if what == "temp_nan": T[0] = np.nan
    if what == "u_one": u[0, k] = 1.0
    if what == "u_neg": u[0, 0] = -0.1
    if what == "nan_logit": draft[0, 1, 3] = np.nan
    if what == "inf_logit": target[0, 2, 0] = np.inf
    if what == "all_neg_inf": target[0, 1, :] = -np.inf
    r = oracle.verify(target, draft, d, u, T)
    assert r.n_accepted[0] == -1 and np.all(r.tokens[0] == -1)
    assert r.n_accepted[1] == 2 and r.errors == 1     # the other sequence is unaffected
