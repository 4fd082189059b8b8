"""Tree verification on the GPU (``spec_verify_tree``) against the oracle's
``verify_tree`` (reading R18 in ``oracle/spec_verify_oracle.c``).

Rule: tokens, counts and accepted nodes bit-exact, except for a sequence with
a decision whose uniform lies within 1e-5 of the oracle's threshold (a tested
child's min(1, R/q), or either CDF point of the final token), which is
counted and left out; R(t_c) and q(t_c) within 1e-5 at every tested child;
error sequences identical.  Child tokens are drawn from the parent's
processed draft row (the oracle's sampler), as the method assumes.
"""
import numpy as np
import pytest

import oracle
import workloads
from paritylib import DECISION_TOL, PROB_TOL, to_dev

pytestmark = pytest.mark.gpu

SHAPES = {
    "chain": lambda N: np.arange(N, dtype=np.int32),
    "binary": lambda N: (np.arange(N, dtype=np.int32)) // 2,
    "star": lambda N: np.zeros(N, dtype=np.int32),
    "mixed": lambda N: np.array([0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 6, 6][:N], dtype=np.int32),
}


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    import __graft_entry__

    __graft_entry__.build()
    return cuda_device


def _tree_case(name, seed, B, N, shape, **over):
    case = workloads.make_case(name, seed=seed, B=B, k=N, **over)
    target = case.target                                       # [B, N+1, V]
    greedy = case.mode == "greedy"
    draft = None if greedy else np.concatenate([case.draft, case.draft[:, -1:]], axis=1)
    parents = np.tile(SHAPES[shape](N), (B, 1))
    if greedy:
        # the proposer's guesses: the argmax of a noisy copy of the parent's target row
        rows = case.draft_proxy  # [B, N, V]: a parent is always below N
        toks = np.stack([[oracle.argmax_row(rows[b, parents[b, n]]) for n in range(N)] for b in range(B)])
        u = None
    else:
        # node n's token is drawn from its parent's processed draft row
        par_rows = np.take_along_axis(draft, parents[:, :, None], axis=1)           # [B, N, V]
        temp_rows = np.repeat(case.temperature, N).reshape(B, N)
        toks = oracle.sample_rows(par_rows, case.draft_uniforms[:, :N], temp_rows.reshape(-1), case.top_k)[0]
        u = case.uniforms
    return case, target, draft, np.asarray(toks, np.int32).reshape(B, N), parents.astype(np.int32), u


def _run(case, target, draft, toks, parents, u, greedy, path="list"):
    import torch

    import draft_token_verification_verify_b200 as sv

    dev = torch.device("cuda:0")
    B, N = toks.shape
    nodes = torch.full((B, N + 1), -7, dtype=torch.int32, device=dev)
    p = torch.full((B, N), 7.0, dtype=torch.float32, device=dev)
    q = torch.full((B, N), 7.0, dtype=torch.float32, device=dev)
    tok, n = sv.verify_tree(to_dev(target), None if greedy else to_dev(draft), torch.from_numpy(toks).to(dev),
                            torch.from_numpy(parents).to(dev), None if greedy else to_dev(u),
                            None if greedy else to_dev(case.temperature), case.top_k, greedy=greedy,
                            out_nodes=nodes, out_p=None if greedy else p, out_q=None if greedy else q,
                            workspace=None if path == "list" else False)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), n.cpu().numpy(), nodes.cpu().numpy(), p.cpu().numpy(), q.cpu().numpy()


def _check(case, target, draft, toks, parents, u, max_flag_frac=0.05, path="list"):
    greedy = case.mode == "greedy"
    ref = oracle.verify_tree(target, draft, toks, parents, u, None if greedy else case.temperature, case.top_k,
                             greedy=greedy)
    tok, n, nodes, p, q = _run(case, target, draft, toks, parents, u, greedy, path)
    B, N = toks.shape
    flagged = exact = 0
    for b in range(B):
        if ref.n_accepted[b] < 0:
            assert n[b] == -1 and np.all(tok[b] == -1), (b, n[b], tok[b])
            continue
        if not greedy:
            tested = np.flatnonzero(~np.isnan(ref.ratio[b]))
            near = any(abs(float(u[b, c]) - ref.ratio[b, c]) < DECISION_TOL for c in tested)
            near |= abs(float(u[b, N]) - ref.cdf_lo[b]) < DECISION_TOL or abs(float(u[b, N]) - ref.cdf_hi[b]) < DECISION_TOL
            if near:
                flagged += 1
                continue
            assert np.array_equal(np.flatnonzero(~np.isnan(p[b])), tested), (b, p[b], ref.p[b])
            assert np.max(np.abs(p[b, tested] - ref.p[b, tested]), initial=0) <= PROB_TOL, (b, p[b], ref.p[b])
            assert np.max(np.abs(q[b, tested] - ref.q[b, tested]), initial=0) <= PROB_TOL, (b, q[b], ref.q[b])
        assert n[b] == ref.n_accepted[b], (b, n[b], ref.n_accepted[b], tok[b], ref.tokens[b])
        assert np.array_equal(tok[b], ref.tokens[b]), (b, tok[b], ref.tokens[b])
        assert np.array_equal(nodes[b], ref.nodes[b]), (b, nodes[b], ref.nodes[b])
        exact += 1
    print(f"sequences {B}: exact {exact}, flagged {flagged}, errors {ref.errors}")
    assert flagged <= max(1, int(max_flag_frac * B)), flagged
    return ref, (tok, n, nodes, p, q)


PATHS = ["list", "rows"]  # the walk on the streaming pass's kept lists, or over the rows


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("shape", ["binary", "star", "mixed"])
def test_batched_top_k_full_vocabulary(shape, path):
    """bf16, V = 151,936, T = 0.7, top-k 50 (the batched workload's value model)."""
    case, t, d, toks, par, u = _tree_case("batched", 91, 16, 9, shape)
    ref, _ = _check(case, t, d, toks, par, u, path=path)
    assert ref.errors == 0


def test_fp32_softmax_mixed_temperatures():
    case, t, d, toks, par, u = _tree_case("large", 92, 8, 7, "binary", V=20011)
    _check(case, t, d, toks, par, u)


def test_single_full_vocabulary_no_top_k():
    case, t, d, toks, par, u = _tree_case("single", 93, 4, 8, "mixed")
    _check(case, t, d, toks, par, u)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("V", [3, 257, 30011])
def test_ragged_and_tiny_vocabularies(V, path):
    case, t, d, toks, par, u = _tree_case("batched", 94, 24, 6, "binary", V=V, top_k=min(5, V - 1))
    _check(case, t, d, toks, par, u, path=path)


def test_chain_trees_match_chain_verification():
    """A chain-shaped tree gives what spec_verify gives for the chain."""
    import torch

    import draft_token_verification_verify_b200 as sv

    case = workloads.make_case("batched", seed=95, B=12, V=30011)
    k = case.k
    drafts = oracle.draft_tokens_for(case)
    dev = torch.device("cuda:0")
    tok_c, n_c = sv.verify(to_dev(case.target), to_dev(case.draft), torch.from_numpy(drafts).to(dev),
                           to_dev(case.uniforms), to_dev(case.temperature), case.top_k)
    d_tree = np.concatenate([case.draft, case.draft[:, -1:]], axis=1)
    par = np.tile(np.arange(k, dtype=np.int32), (case.B, 1))
    tok_t, n_t = sv.verify_tree(to_dev(case.target), to_dev(d_tree), torch.from_numpy(drafts).to(dev),
                                torch.from_numpy(par).to(dev), to_dev(case.uniforms), to_dev(case.temperature),
                                case.top_k)
    torch.cuda.synchronize()
    ref = oracle.verify(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k)
    for b in range(case.B):
        j = ref.n_accepted[b]
        u = case.uniforms[b]
        if any(abs(float(u[i]) - ref.ratio[b, i]) < DECISION_TOL for i in range(min(j + 1, k))) or \
                abs(float(u[k]) - ref.cdf_lo[b]) < DECISION_TOL or abs(float(u[k]) - ref.cdf_hi[b]) < DECISION_TOL:
            continue
        assert np.array_equal(tok_t[b].cpu().numpy(), tok_c[b].cpu().numpy()), b
        assert int(n_t[b]) == int(n_c[b]) == j


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("shape", ["binary", "star"])
def test_greedy_trees(shape, path):
    case, t, d, toks, par, u = _tree_case("greedy", 96, 32, 7, shape, V=30011)
    ref, _ = _check(case, t, d, toks, par, u, path=path)
    assert ref.errors == 0


def test_overflowing_kept_list_falls_back_to_the_rows():
    """3,000 tied maxima in one target row: its kept list cannot hold them,
    the list walk leaves the sequence to the walk over the rows."""
    case, t, d, toks, par, u = _tree_case("batched", 99, 6, 4, "binary", V=30011)
    t = t.copy()
    row = t[2, 0]
    top = row[np.argmax((row.astype(np.uint32) << 16).view(np.float32))]  # bf16 bits of the row maximum
    t[2, 0, :3000] = top
    ref, _ = _check(case, t, d, toks, par, u, path="list")
    assert ref.n_accepted[2] >= 0


@pytest.mark.parametrize("path", PATHS)
def test_row_errors(path):
    case, t, d, toks, par, u = _tree_case("batched", 97, 6, 4, "binary", V=4099)
    t = t.copy()
    toks = toks.copy()
    par = par.copy()
    u = u.copy()
    toks[0, 1] = case.V          # token outside [0, V)
    par[1, 2] = 3                # parent not before its child
    par[2, 0] = -1               # parent outside [0, n)
    u[3, 1] = 1.0                # uniform outside [0, 1)
    t[4, 0, 7] = 0x7fc0          # bf16 NaN in the root's target row (always read)
    ref, (tok, n, *_rest) = _check(case, t, d, toks, par, u, path=path)
    assert list(ref.n_accepted[:5]) == [-1] * 5 and list(n[:5]) == [-1] * 5
    assert ref.n_accepted[5] >= 0 and n[5] >= 0


def test_repeated_calls_agree():
    case, t, d, toks, par, u = _tree_case("batched", 98, 8, 9, "mixed", V=30011)
    a = _run(case, t, d, toks, par, u, False)
    b = _run(case, t, d, toks, par, u, False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y, equal_nan=True)
