"""Pins of the oracle's tree verification (reading R18 in
``oracle/spec_verify_oracle.c``; candidate trees are named in section
"提议方式与实现形态", paragraph 3, of the entry "推测解码", the chain rule is
section "提议与核验的基本步骤", paragraphs 2-4).

- the worked example of paragraph 3 as one- and two-child trees, by hand;
- a chain-shaped tree gives exactly what the chain verification gives
  (tokens, counts, p and q), stochastic and greedy, bf16 and fp32, with top-k
  and temperature;
- with every node's children drawn independently from the node's draft row,
  the first emitted token follows the root's target row and the token after
  an accepted child follows that child's target row (chi-square, the law
  that makes the walk a valid sampler);
- a rejection whose residual has no mass leaves the current distribution;
- greedy trees and row errors by hand.
"""
import numpy as np
import pytest
from scipy import stats

import oracle

WORKED_P = np.log(np.array([0.6, 0.3, 0.1]))
WORKED_Q = np.log(np.array([0.5, 0.4, 0.1]))


def _rows(*rows, dtype=np.float32):
    return np.stack(rows).astype(dtype)[None]


def test_worked_example_one_child():
    t = _rows(WORKED_P, WORKED_P)
    d = _rows(WORKED_Q, WORKED_Q)
    acc = oracle.verify_tree(t, d, [[1]], [[0]], np.array([[0.7499, 0.5]], np.float32))
    assert acc.n_accepted[0] == 1 and list(acc.tokens[0]) == [1, 0]  # B accepted, bonus A (0.5 < 0.6)
    assert abs(acc.ratio[0, 0] - 0.75) < 1e-6
    rej = oracle.verify_tree(t, d, [[1]], [[0]], np.array([[0.7501, 0.99]], np.float32))
    assert rej.n_accepted[0] == 0 and list(rej.tokens[0]) == [0, -1]  # the residual is all on A


def test_worked_example_two_children():
    # root children B then B: after B is rejected the current distribution is
    # (1, 0, 0); the second B has probability 0 there and is rejected too;
    # the residual of (1,0,0) against q is (0.5,0,0), normalised all on A
    t = _rows(WORKED_P, WORKED_P, WORKED_P)
    d = _rows(WORKED_Q, WORKED_Q, WORKED_Q)
    r = oracle.verify_tree(t, d, [[1, 1]], [[0, 0]], np.array([[0.9, 0.0, 0.3]], np.float32))
    assert r.n_accepted[0] == 0 and list(r.tokens[0]) == [0, -1, -1]
    assert abs(r.p[0, 1]) < 1e-12 and abs(r.q[0, 1] - 0.4) < 1e-6 and r.ratio[0, 1] == 0.0
    # children B then A: A has current probability 1 > u * 0.5 for every u, so it is accepted
    r = oracle.verify_tree(t, d, [[1, 0]], [[0, 0]], np.array([[0.9, 0.999, 0.5]], np.float32))
    assert r.n_accepted[0] == 1 and list(r.tokens[0][:2]) == [0, 0] and r.nodes[0, 0] == 2
    assert abs(r.p[0, 1] - 1.0) < 1e-12 and abs(r.q[0, 1] - 0.5) < 1e-6


def _random_case(rng, B, k, V, dtype, scale=2.0):
    t = (rng.normal(0, scale, (B, k + 1, V))).astype(np.float32)
    d = (t[:, : k] + rng.normal(0, 1.0, (B, k, V))).astype(np.float32)
    if dtype == "bf16":
        to_bf16 = lambda a: (a.view(np.uint32) + 0x8000 >> 16).astype(np.uint16)
        return to_bf16(t), to_bf16(d)
    return t, d


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("top_k", [0, 3])
def test_chain_trees_equal_chain_verification(dtype, top_k):
    rng = np.random.default_rng(7)
    B, k, V = 400, 4, 9
    t, d = _random_case(rng, B, k, V, dtype)
    temp = rng.choice(np.array([0.5, 1.0, 1.5], np.float32), B)
    u = rng.random((B, k + 1), dtype=np.float32)
    toks = oracle.sample_rows(d, rng.random((B, k), dtype=np.float32), np.repeat(temp, k), top_k)[0]
    toks = np.asarray(toks, np.int32).reshape(B, k)
    chain = oracle.verify(t, d, toks, u, temp, top_k)
    # the tree carries one more draft row (the leaf's, never read)
    d_tree = np.concatenate([d, d[:, -1:]], axis=1)
    parents = np.tile(np.arange(k, dtype=np.int32), (B, 1))  # node n's parent is n - 1
    tree = oracle.verify_tree(t, d_tree, toks, parents, u, temp, top_k)
    assert np.array_equal(tree.n_accepted, chain.n_accepted)
    assert np.array_equal(tree.tokens, chain.tokens)
    for b in range(B):
        j = chain.n_accepted[b]
        tested = min(j + 1, k)
        assert np.allclose(tree.p[b, :tested], chain.p[b, :tested], rtol=0, atol=1e-15)
        assert np.allclose(tree.q[b, :tested], chain.q[b, :tested], rtol=0, atol=1e-15)
        assert np.all(np.isnan(tree.p[b, tested:]))
        assert list(tree.nodes[b, :j]) == list(range(1, j + 1))
    greedy_chain = oracle.verify(t, None, toks, None, None, 0, greedy=True)
    greedy_tree = oracle.verify_tree(t, None, toks, parents, greedy=True)
    assert np.array_equal(greedy_tree.tokens, greedy_chain.tokens)
    assert np.array_equal(greedy_tree.n_accepted, greedy_chain.n_accepted)


def _chi2_pvalue(counts, probs):
    counts = np.asarray(counts, np.float64)
    exp = probs * counts.sum()
    keep = exp >= 5
    c = np.append(counts[keep], counts[~keep].sum())
    e = np.append(exp[keep], exp[~keep].sum())
    if e[-1] == 0:
        c, e = c[:-1], e[:-1]
    return stats.chisquare(c, e).pvalue


@pytest.mark.parametrize("top_k,T", [(0, 1.0), (3, 0.7)])
def test_emitted_law_of_branching_trees(top_k, T):
    """Root with three children, each with two children; every node's
    children are drawn independently from the node's processed draft row."""
    rng = np.random.default_rng(11 + top_k)
    V, N, B = 6, 9, 300_000
    parents = np.array([0, 0, 0, 1, 1, 2, 2, 3, 3], np.int32)
    base_t = rng.normal(0, 1.5, (N + 1, V)).astype(np.float32)
    base_d = (base_t + rng.normal(0, 1.0, (N + 1, V))).astype(np.float32)
    P = np.stack([oracle.process_row(base_t[n], T, top_k) for n in range(N + 1)])
    Q = np.stack([oracle.process_row(base_d[n], T, top_k) for n in range(N + 1)])
    toks = np.empty((B, N), np.int32)
    for c in range(1, N + 1):
        a = parents[c - 1]
        toks[:, c - 1] = rng.choice(V, size=B, p=Q[a] / Q[a].sum())
    u = rng.random((B, N + 1), dtype=np.float32)
    t = np.broadcast_to(base_t, (B, N + 1, V))
    d = np.broadcast_to(base_d, (B, N + 1, V))
    temp = np.full(B, T, np.float32)
    r = oracle.verify_tree(t, d, toks, np.tile(parents, (B, 1)), u, temp, top_k)
    assert r.errors == 0
    first = r.tokens[:, 0]
    assert _chi2_pvalue(np.bincount(first, minlength=V), P[0]) > 1e-3
    for c in (1, 2, 3):  # after an accepted child, the next token follows its target row
        sel = r.nodes[:, 0] == c
        assert sel.sum() > 2_000
        assert _chi2_pvalue(np.bincount(r.tokens[sel, 1], minlength=V), P[c]) > 1e-3


def test_zero_residual_keeps_the_current_distribution():
    # p = q, and the child's token has probability 0 on both sides: it is
    # rejected (u * 0 < 0 fails), max(0, p - q) has no mass, so the final token
    # is drawn from p itself (the reading of R8 on a tree)
    row = np.array([0.0, 1.0, -np.inf, 0.5], np.float32)
    t = _rows(row, row)
    d = _rows(row, row)
    r = oracle.verify_tree(t, d, [[2]], [[0]], np.array([[0.3, 0.6]], np.float32))
    assert r.n_accepted[0] == 0
    w = oracle.process_row(row)
    y = int(np.argmax(np.cumsum(w) > 0.6))
    assert r.tokens[0, 0] == y


def test_greedy_tree_by_hand():
    root = np.array([0.0, 3.0, 1.0, 3.0], np.float32)  # argmax 1 (lowest index of the tie)
    n1 = np.array([5.0, 0.0, 0.0, 0.0], np.float32)   # argmax 0
    n2 = np.array([0.0, 0.0, 0.0, 9.0], np.float32)   # argmax 3
    n3 = np.array([0.0, 0.0, 7.0, 0.0], np.float32)   # argmax 2
    t = _rows(root, n1, n2, n3)
    # node 1 (token 3) and node 2 (token 1) under the root: node 2 matches the argmax;
    # node 3 (token 0) under node 2: no match there is 3, so 3 is emitted
    r = oracle.verify_tree(t, None, [[3, 1, 0]], [[0, 0, 2]], greedy=True)
    assert r.n_accepted[0] == 1 and list(r.tokens[0]) == [1, 3, -1, -1] and r.nodes[0, 0] == 2


def test_row_errors():
    rng = np.random.default_rng(3)
    V, N = 5, 3
    t = rng.normal(0, 1, (6, N + 1, V)).astype(np.float32)
    d = rng.normal(0, 1, (6, N + 1, V)).astype(np.float32)
    toks = np.zeros((6, N), np.int32)
    par = np.tile(np.array([0, 0, 1], np.int32), (6, 1))
    u = np.full((6, N + 1), 0.5, np.float32)
    toks[0, 1] = V            # token outside [0, V)
    par[1, 2] = 3             # parent not before its child
    par[2, 0] = -1            # parent outside [0, n)
    u[3, 2] = 1.0             # uniform outside [0, 1)
    t[4, 0, 2] = np.nan       # the root's target row: always read
    # sequence 5: node 1's token has probability 0 at the root, so node 1 is
    # never accepted and node 3 (its child) never visited: its rows are not read
    toks[5, 0] = 4
    t[5, 0, 4] = -np.inf
    t[5, 3, 1] = np.nan
    d[5, 3, 1] = np.nan
    r = oracle.verify_tree(t, d, toks, par, u)
    assert list(r.n_accepted[:5]) == [-1] * 5
    assert np.all(r.tokens[:5] == -1)
    assert r.n_accepted[5] >= 0  # the bad row is never read
