"""Pins of the oracle's output projection and the greedy verification on its
logits (``oracle_head_logits`` and ``verify_head_greedy``; the target's one
forward pass, section "提议与核验的基本步骤", paragraph 1, of the entry
"推测解码"; the greedy rule, paragraph 4).

- the logits against exact rational arithmetic on the bf16 values (every bf16
  value is a dyadic rational), within the textbook bound of recursive
  summation in double;
- integer-valued inputs, where every partial sum is exact: equality;
- one-hot weight rows pick the hidden entries; a negated weight negates the
  logits;
- the greedy chain on fp64 logits equals the chain on the same values given as
  float32 rows (the pinned float32 path), and a small case worked by hand;
- a NaN hidden entry makes its sequence a row error.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def bf16_bits(a):
    """Round-to-nearest-even float32 -> bf16 bit patterns (finite inputs)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bf16_value(bits):
    return float((np.uint32(bits) << np.uint32(16)).view(np.float32))


def test_logits_match_exact_rational_sums():
    rng = np.random.default_rng(1)
    R, V, H = 3, 11, 37
    h = bf16_bits(rng.normal(0, 1, (R, H)))
    w = bf16_bits(rng.normal(0, 0.3, (V, H)))
    z, a = oracle.head_logits(h, w)
    u = 2.0 ** -53
    for r in range(R):
        for v in range(V):
            terms = [Fraction(bf16_value(h[r, j])) * Fraction(bf16_value(w[v, j])) for j in range(H)]
            exact = sum(terms)
            mag = sum(abs(t) for t in terms)
            bound = H * u / (1 - H * u) * float(mag)
            assert abs(Fraction(z[r, v]) - exact) <= Fraction(bound), (r, v)
            assert abs(Fraction(a[r, v]) - mag) <= Fraction(bound), (r, v)


def test_integer_inputs_are_exact():
    rng = np.random.default_rng(2)
    R, V, H = 4, 9, 64
    hv = rng.integers(-8, 9, (R, H)).astype(np.float32)
    wv = rng.integers(-8, 9, (V, H)).astype(np.float32)
    z, a = oracle.head_logits(bf16_bits(hv), bf16_bits(wv))
    exact = hv.astype(np.int64) @ wv.astype(np.int64).T
    assert np.array_equal(z, exact.astype(np.float64))
    assert np.array_equal(a, (np.abs(hv).astype(np.int64) @ np.abs(wv).astype(np.int64).T).astype(np.float64))


def test_one_hot_rows_pick_hidden_entries_and_negation_negates():
    rng = np.random.default_rng(3)
    R, H = 5, 24
    V = H
    perm = rng.permutation(H)
    h = bf16_bits(rng.normal(0, 2, (R, H)))
    w = np.zeros((V, H), dtype=np.uint16)
    w[np.arange(V), perm] = 0x3F80  # 1.0
    z, _ = oracle.head_logits(h, w)
    hv = (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(z, hv[:, perm])
    w2 = bf16_bits(rng.normal(0, 1, (V, H)))
    z2, _ = oracle.head_logits(h, w2)
    zn, _ = oracle.head_logits(h, w2 ^ np.uint16(0x8000))
    assert np.array_equal(zn, -z2)


def test_row_range_matches_the_full_computation():
    rng = np.random.default_rng(4)
    h = bf16_bits(rng.normal(0, 1, (6, 16)))
    w = bf16_bits(rng.normal(0, 1, (7, 16)))
    z, a = oracle.head_logits(h, w)
    z2, a2 = oracle.head_logits(h, w, 2, 3)
    assert np.array_equal(z2, z[2:5]) and np.array_equal(a2, a[2:5])


@pytest.mark.parametrize("seed", [5, 6])
def test_greedy_on_f64_logits_equals_the_float32_path(seed):
    """Integer-valued logits are exact in float32 and fp64 alike: the greedy
    chain read from the fp64 rows equals the one read from float32 rows."""
    rng = np.random.default_rng(seed)
    B, k, V, H = 300, 4, 7, 8
    h = bf16_bits(rng.integers(-3, 4, (B, k + 1, H)).astype(np.float32))
    w = bf16_bits(rng.integers(-3, 4, (V, H)).astype(np.float32))
    z, _ = oracle.head_logits(h, w)
    z = z.reshape(B, k + 1, V)
    g = z.argmax(axis=-1)
    drafts = np.where(rng.random((B, k)) < 0.7, g[:, :k], rng.integers(0, V, (B, k))).astype(np.int32)
    hr = oracle.verify_head_greedy(h, w, drafts)
    ref = oracle.verify(z.astype(np.float32), None, drafts, None, greedy=True)
    assert np.array_equal(hr.result.tokens, ref.tokens)
    assert np.array_equal(hr.result.n_accepted, ref.n_accepted)
    assert np.array_equal(hr.z, z)
    assert 0 < np.mean(ref.n_accepted == k) < 1  # both outcomes occur


def test_greedy_worked_by_hand():
    one, two, neg = 0x3F80, 0x4000, 0xBF80  # 1.0, 2.0, -1.0
    # H = 2; weight rows: [1, 0], [0, 1], [1, 1], [-1, 0]
    w = np.array([[one, 0], [0, one], [one, one], [neg, 0]], dtype=np.uint16)
    # positions: h = [2, -1] -> z = [2, -1, 1, -2] (argmax 0)
    #            h = [1, 1]  -> z = [1, 1, 2, -1]  (argmax 2)
    #            h = [-1, 2] -> z = [-1, 2, 1, 1]  (argmax 1)
    h = np.array([[[two, neg], [one, one], [neg, two]]], dtype=np.uint16)
    r = oracle.verify_head_greedy(h, w, np.array([[0, 2]])).result
    assert r.n_accepted[0] == 2 and list(r.tokens[0]) == [0, 2, 1]  # both match, bonus 1
    r = oracle.verify_head_greedy(h, w, np.array([[0, 1]])).result
    assert r.n_accepted[0] == 1 and list(r.tokens[0]) == [0, 2, -1]  # mismatch at 1: emit 2
    r = oracle.verify_head_greedy(h, w, np.array([[3, 2]])).result
    assert r.n_accepted[0] == 0 and list(r.tokens[0]) == [0, -1, -1]


def test_nan_hidden_entry_is_a_row_error():
    rng = np.random.default_rng(7)
    B, k, V, H = 3, 2, 5, 8
    h = bf16_bits(rng.normal(0, 1, (B, k + 1, H)))
    w = bf16_bits(rng.normal(0, 1, (V, H)))
    h[1, 2, 3] = 0x7FC0  # NaN in the bonus position's hidden state of sequence 1
    r = oracle.verify_head_greedy(h, w, np.zeros((B, k), np.int32)).result
    assert r.n_accepted[1] == -1 and np.all(r.tokens[1] == -1)
    assert r.n_accepted[0] >= 0 and r.n_accepted[2] >= 0


def test_sequence_subset():
    rng = np.random.default_rng(8)
    B, k, V, H = 5, 3, 6, 16
    h = bf16_bits(rng.normal(0, 1, (B, k + 1, H)))
    w = bf16_bits(rng.normal(0, 1, (V, H)))
    d = rng.integers(0, V, (B, k)).astype(np.int32)
    full = oracle.verify_head_greedy(h, w, d)
    sub = oracle.verify_head_greedy(h, w, d, seqs=[4, 1], threads=2)
    assert np.array_equal(sub.result.tokens, full.result.tokens[[4, 1]])
    assert np.array_equal(sub.z, full.z[[4, 1]])
