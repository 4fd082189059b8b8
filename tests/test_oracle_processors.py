"""Pins of the oracle's further logits processors (readings R12..R15 in
``oracle/spec_verify_oracle.c``): repetition penalty, vocabulary mask and
nucleus (top-p), which the speculative decoding entry "推测解码" (section
"提议与核验的基本步骤", paragraph 4) lists among the processing rules that
must act identically on the target and the draft distributions.

Expected values come from closed forms computed here with numpy, hand cases,
invariants and a brute-force enumeration of the output law; none of them
calls the oracle to produce its own expectation.
"""
import itertools

import numpy as np
import pytest

import oracle


def softmax(z, T=1.0):
    z = np.asarray(z, dtype=np.float64) / T
    m = np.max(z[np.isfinite(z)])
    e = np.where(np.isfinite(z), np.exp(z - m), 0.0)
    return e / e.sum()


def f32(x):
    return np.asarray(x, dtype=np.float32)


# --------------------------------------------------------------------------
# repetition penalty (R13)
# --------------------------------------------------------------------------

def test_repetition_penalty_closed_form():
    z = f32([2.0, -1.0, 0.5, 0.0])
    got = oracle.process_row_procs(z, rep_penalty=2.0, rep_ids=[0, 1])
    assert np.allclose(got, softmax([1.0, -2.0, 0.5, 0.0]), rtol=0, atol=1e-15)


def test_repetition_penalty_each_id_once_and_out_of_range_ignored():
    z = f32([1.5, 0.25, -0.75, 3.0])
    once = oracle.process_row_procs(z, rep_penalty=1.7, rep_ids=[2])
    many = oracle.process_row_procs(z, rep_penalty=1.7, rep_ids=[2, 2, 9, -1, 2])
    assert np.array_equal(once, many)
    penalised = float(np.float32(-0.75 * 1.7))  # the exact product, rounded once to fp32
    assert np.allclose(once, softmax([1.5, 0.25, penalised, 3.0]), rtol=0, atol=1e-15)


def test_repetition_penalty_rounds_to_fp32():
    """The penalised logit is the correctly rounded fp32 quotient (product):
    1.5 / 1.2f rounds up to exactly 1.25 in fp32 while its fp64 value lies just
    below, so a competitor at 1.25 ties with the penalised token at top-1 and
    both are kept; unrounded, top-1 would keep the competitor alone.  Likewise
    -1.5 * 1.2f against its own fp32 rounding."""
    theta = np.float32(1.2)
    c = np.float32(1.5) / theta                      # numpy fp32 division is IEEE round-to-nearest
    assert float(c) == 1.25 and 1.5 / float(theta) < 1.25  # the rounding matters for this pair
    z = f32([1.5, c, -3.0])
    got = oracle.process_row_procs(z, top_k=1, rep_penalty=float(theta), rep_ids=[0])
    assert np.allclose(got, [0.5, 0.5, 0.0], rtol=0, atol=1e-15)
    neg = oracle.process_row_procs(f32([-1.5, np.float32(-1.5) * theta, -9.0]), top_k=1,
                                   rep_penalty=float(theta), rep_ids=[0])
    assert np.allclose(neg, [0.5, 0.5, 0.0], rtol=0, atol=1e-15)


def test_unit_penalty_and_no_processor_equal_plain_processing():
    rng = np.random.default_rng(5)
    for _ in range(20):
        z = f32(rng.normal(0, 2, 50))
        T = float(rng.uniform(0.4, 1.8))
        K = int(rng.integers(0, 50))
        plain = oracle.process_row(z, T, K)
        assert np.array_equal(oracle.process_row_procs(z, T, K), plain)
        assert np.array_equal(oracle.process_row_procs(z, T, K, rep_penalty=1.0, rep_ids=[1, 2, 3]), plain)


# --------------------------------------------------------------------------
# vocabulary mask (R14)
# --------------------------------------------------------------------------

def test_mask_allows_listed_tokens_only():
    z = f32(np.zeros(40))
    got = oracle.process_row_procs(z, mask=oracle.allow_mask(40, [1, 33]))
    want = np.zeros(40)
    want[[1, 33]] = 0.5
    assert np.array_equal(got, want)


def test_mask_bit_layout_word_boundaries():
    V = 70
    z = f32(np.arange(V) * 0.01)
    for v in (0, 31, 32, 63, 64, 69):
        got = oracle.process_row_procs(z, mask=oracle.allow_mask(V, [v]))
        assert got[v] == 1.0 and got.sum() == 1.0


@pytest.mark.parametrize("theta", [0.0, -1.5, float("nan"), float("inf")])
def test_penalty_not_positive_and_finite_is_a_row_error(theta):
    """Reading R13: theta must be finite and > 0, listed ids or not."""
    z = f32([0.5, 1.0, 2.0])
    assert oracle.process_row_procs(z, rep_penalty=theta, rep_ids=[1]) is None
    assert oracle.process_row_procs(z, rep_penalty=theta) is None
    assert oracle.process_row_procs(z, rep_penalty=2.0, rep_ids=[1]) is not None


def test_everything_masked_is_a_row_error():
    assert oracle.process_row_procs(f32([0.0, 1.0, 2.0]), mask=oracle.allow_mask(3, [])) is None


def test_mask_then_top_k():
    # the mask acts before top-k: the best allowed tokens fill the K slots
    z = f32([5.0, 4.0, 3.0, 2.0, 1.0])
    got = oracle.process_row_procs(z, top_k=2, mask=oracle.allow_mask(5, [1, 3, 4]))
    assert np.allclose(got, [0, softmax([4.0, 2.0])[0], 0, softmax([4.0, 2.0])[1], 0], rtol=0, atol=1e-15)


def test_penalty_before_top_k():
    # R12: the penalty changes which token survives top-1
    z = f32([3.0, 2.9, 1.0])
    assert np.array_equal(oracle.process_row_procs(z, top_k=1), [1.0, 0.0, 0.0])
    assert np.array_equal(oracle.process_row_procs(z, top_k=1, rep_penalty=2.0, rep_ids=[0]), [0.0, 1.0, 0.0])


# --------------------------------------------------------------------------
# nucleus (R15)
# --------------------------------------------------------------------------

def _quarters():
    # probabilities 0.5, 0.25, 0.125, 0.125 (up to the log/exp round trip)
    return f32(np.log([4.0, 2.0, 1.0, 1.0]))


@pytest.mark.parametrize("top_p,kept", [(0.3, [0]), (0.7, [0, 1]), (0.8, [0, 1, 2, 3]), (0.95, [0, 1, 2, 3]),
                                        (1.0, [0, 1, 2, 3])])
def test_nucleus_hand_cases(top_p, kept):
    got = oracle.process_row_procs(_quarters(), top_p=top_p)
    base = softmax(_quarters())
    want = np.zeros(4)
    want[kept] = base[kept] / base[kept].sum()
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_nucleus_keeps_ties_at_the_cut():
    # 0.4, 0.3, 0.3: the running sum reaches 0.5 at a 0.3, so both 0.3s stay
    z = f32(np.log([0.4, 0.3, 0.3]))
    got = oracle.process_row_procs(z, top_p=0.5)
    assert np.count_nonzero(got) == 3


def test_nucleus_after_temperature():
    # a flatter distribution (higher T) needs more tokens for the same mass
    z = f32([2.0, 1.0, 0.0, -1.0])
    cold = oracle.process_row_procs(z, 0.5, top_p=0.9)
    hot = oracle.process_row_procs(z, 3.0, top_p=0.9)
    assert np.count_nonzero(cold) < np.count_nonzero(hot)
    for T, got in ((0.5, cold), (3.0, hot)):
        base = softmax(z, T)
        order = np.argsort(-base, kind="stable")
        c = np.cumsum(base[order])
        cut = base[order][np.argmax(c >= 0.9)]
        want = np.where(base >= cut, base, 0.0)
        assert np.allclose(got, want / want.sum(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(12))
def test_nucleus_invariants_random_rows(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(2, 300))
    z = f32(np.round(rng.normal(0, 2, V), 1))  # rounding makes ties common
    T = float(rng.uniform(0.5, 1.5))
    K = int(rng.integers(0, V + 1))
    top_p = float(rng.uniform(0.05, 0.99))
    base = oracle.process_row(z, T, K)
    got = oracle.process_row_procs(z, T, K, top_p=top_p)
    kept = got > 0
    assert kept.any() and np.isclose(got.sum(), 1.0, rtol=0, atol=1e-12)
    # kept tokens are exactly those at or above a cut value, and keep their ratios
    assert base[kept].min() >= base[~kept].max(initial=0.0)
    ratio = got[kept] / base[kept]
    assert np.allclose(ratio, ratio[0], rtol=1e-12, atol=0)
    # the kept mass reaches top_p; without the smallest kept value it does not
    mass = base[kept].sum()
    assert mass >= top_p - 1e-12
    low = base[kept].min()
    assert base[kept & (base > low)].sum() < top_p + 1e-12


# --------------------------------------------------------------------------
# verification with processors
# --------------------------------------------------------------------------

def test_verify_without_processors_equals_plain_verify():
    rng = np.random.default_rng(3)
    B, k, V = 16, 3, 60
    target = f32(rng.normal(0, 2, (B, k + 1, V)))
    draft = f32(target[:, :k] + rng.normal(0, 1, (B, k, V)))
    temp = f32(rng.uniform(0.5, 1.5, B))
    u = f32(rng.uniform(0, 1, (B, k + 1)))
    drafts = oracle.sample_rows(draft, u[:, :k], np.repeat(temp, k), 10)[0].astype(np.int32)
    a = oracle.verify(target, draft, drafts, u, temp, 10)
    b = oracle.verify_procs(target, draft, drafts, u, temp, 10)
    for f in ("tokens", "n_accepted", "p", "q", "cdf_lo", "cdf_hi"):
        assert np.array_equal(getattr(a, f), getattr(b, f), equal_nan=True), f


def test_verify_rejects_a_draft_token_the_target_nucleus_drops():
    """Reading R1 (accept iff u*q < p) with the nucleus in effect: the target
    keeps only token 0 (p(1) = 0), the draft only token 1 (q(1) = 1), so even
    u = 0 rejects token 1, and the residual max(0, p - q) is all on token 0."""
    target = f32([[[5, 0, 0], [0, 0, 0]]])
    draft = f32([[[0, 5, 0]]])
    r = oracle.verify_procs(target, draft, np.array([[1]]), f32([[0.0, 0.5]]), top_p=0.5)
    assert r.p[0, 0] == 0.0 and r.q[0, 0] == 1.0
    assert r.n_accepted[0] == 0 and r.tokens[0].tolist() == [0, -1]


@pytest.mark.parametrize("where", ["accept", "final", "negative"])
def test_verify_procs_uniform_out_of_range_is_a_row_error(where):
    """Reading R7: a uniform outside [0, 1) makes its sequence a row error; the
    other sequence is unaffected."""
    V, k = 5, 2
    target = np.zeros((2, k + 1, V), np.float32)
    draft = np.zeros((2, k, V), np.float32)
    u = np.full((2, k + 1), 0.5, np.float32)
    u[0, {"accept": 0, "final": k, "negative": 1}[where]] = -0.1 if where == "negative" else 1.0
    r = oracle.verify_procs(target, draft, np.ones((2, k), np.int32), u, top_p=0.9)
    assert r.n_accepted[0] == -1 and np.all(r.tokens[0] == -1)
    assert r.n_accepted[1] == k and r.errors == 1


def test_each_sequence_uses_its_own_processors():
    """Sequences are verified independently: a batch with different top_p,
    penalties and masks per sequence gives, for every sequence, what that
    sequence gives alone."""
    rng = np.random.default_rng(21)
    B, k, V = 5, 3, 70
    target = f32(rng.normal(0, 2, (B, k + 1, V)))
    draft = f32(target[:, :k] + rng.normal(0, 1, (B, k, V)))
    temp = f32(rng.uniform(0.6, 1.4, B))
    u = f32(rng.uniform(0, 1, (B, k + 1)))
    top_p = f32(rng.uniform(0.5, 0.95, B))
    pen = f32(rng.uniform(0.5, 2.0, B))
    ids = rng.integers(0, V, (B, 6)).astype(np.int32)
    mask = np.stack([oracle.allow_mask(V, rng.choice(V, 40, replace=False)) for _ in range(B)])
    drafts = np.stack([oracle.sample_rows_procs(draft[b:b + 1], u[b:b + 1, :k], np.full(k, temp[b]), 0,
                                                top_p=top_p[b:b + 1], rep_penalty=pen[b:b + 1],
                                                rep_ids=ids[b:b + 1], mask=mask[b:b + 1])[0]
                       for b in range(B)]).astype(np.int32)
    both = oracle.verify_procs(target, draft, drafts, u, temp, 0, top_p=top_p, rep_penalty=pen,
                               rep_ids=ids, mask=mask)
    assert both.errors == 0

    def alone(b, s):
        return oracle.verify_procs(target[b:b + 1], draft[b:b + 1], drafts[b:b + 1], u[b:b + 1],
                                   temp[b:b + 1], 0, top_p=top_p[s:s + 1], rep_penalty=pen[s:s + 1],
                                   rep_ids=ids[s:s + 1], mask=mask[s:s + 1])

    for b in range(B):
        one = alone(b, b)
        for f in ("tokens", "n_accepted", "p", "q", "cdf_lo", "cdf_hi"):
            assert np.array_equal(getattr(both, f)[b], getattr(one, f)[0], equal_nan=True), (b, f)
    # the processors differ enough between sequences to change the results
    assert any(not np.array_equal(alone(b, 0).p, alone(b, b).p, equal_nan=True) for b in range(1, B))


def _pieces(points):
    pts = sorted(set([0.0, 1.0] + [float(x) for x in points if 0.0 < x < 1.0]))
    return [(a, b) for a, b in zip(pts[:-1], pts[1:]) if b - a > 1e-6]


@pytest.mark.parametrize("V,k", [(3, 1), (4, 1), (4, 2)])
@pytest.mark.parametrize("procs", [dict(top_p=0.7), dict(rep_penalty=1.8, rep_ids=[[1]]),
                                   dict(mask=[[0b1011]]),
                                   dict(top_p=0.8, rep_penalty=0.6, rep_ids=[[0, 2]], mask=[[0b1110]])])
@pytest.mark.parametrize("seed", [0, 1])
def test_processors_preserve_the_processed_target_law(V, k, procs, seed):
    """Exact law of the emitted tokens by enumeration: with the processors in
    effect on both sides, emitted[m] | n >= m follows the PROCESSED target
    distribution of position m (the property the method is built to keep)."""
    rng = np.random.default_rng(100 * V + 10 * k + seed)
    T = 0.9
    target = f32(rng.normal(0, 1.5, (k + 1, V)))
    draft = f32(target[:k] + rng.normal(0, 1.0, (k, V)))
    row_procs = {key: (np.asarray(v).ravel() if key in ("rep_ids", "mask") else v) for key, v in procs.items()}
    if "mask" in row_procs:
        row_procs["mask"] = row_procs["mask"].astype(np.uint32)
    p = [oracle.process_row_procs(target[i], T, 0, **row_procs) for i in range(k + 1)]
    q = [oracle.process_row_procs(draft[i], T, 0, **row_procs) for i in range(k)]
    assert all(x is not None for x in p + q)
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
        slots = [_pieces([min(1.0, p[i][d[i]] / q[i][d[i]])]) for i in range(k)]
        for acc in itertools.product(*slots):
            for f in fin:
                rows.append((d, [0.5 * (a + b) for a, b in acc] + [0.5 * (f[0] + f[1])]))
                weights.append(wd * np.prod([b - a for a, b in acc]) * (f[1] - f[0]))
    B = len(rows)
    tk = np.array([r[0] for r in rows], np.int32).reshape(B, k)
    uu = np.array([r[1] for r in rows], np.float32)
    seq = {}
    if "top_p" in procs:
        seq["top_p"] = procs["top_p"]
    if "rep_penalty" in procs:
        seq["rep_penalty"] = procs["rep_penalty"]
        seq["rep_ids"] = np.repeat(np.asarray(procs["rep_ids"], np.int32), B, 0)
    if "mask" in procs:
        seq["mask"] = np.repeat(np.asarray(procs["mask"], np.uint32), B, 0)
    res = oracle.verify_procs(np.repeat(target[None], B, 0), np.repeat(draft[None], B, 0), tk, uu,
                              np.full(B, T, np.float32), 0, **seq)
    assert res.errors == 0
    wts = np.array(weights)
    tol = 1e-9 + abs(1.0 - wts.sum())
    n = res.n_accepted
    for m in range(k + 1):
        reach = n >= m
        P_reach = wts[reach].sum()
        law = np.array([wts[reach & (res.tokens[:, m] == v)].sum() for v in range(V)])
        assert np.allclose(law / P_reach, p[m], rtol=0, atol=tol / max(P_reach, 1e-300)), (m, law / P_reach, p[m])


def test_proposer_draw_with_processors_stays_in_the_kept_set():
    rng = np.random.default_rng(9)
    B, rps, V = 8, 3, 80
    logits = f32(rng.normal(0, 2, (B, rps, V)))
    u = f32(rng.uniform(0, 1, (B, rps)))
    allowed = [rng.choice(V, 20, replace=False) for _ in range(B)]
    mask = np.stack([oracle.allow_mask(V, a) for a in allowed])
    tok = oracle.sample_rows_procs(logits, u, top_p=0.6, mask=mask)
    for b in range(B):
        for r in range(rps):
            prob = oracle.process_row_procs(logits[b, r], 1.0, 0, top_p=0.6, mask=mask[b])
            assert tok[b, r] in set(allowed[b].tolist()) and prob[tok[b, r]] > 0
