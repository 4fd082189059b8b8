"""Nucleus (top-p) on the top-k path: the CUDA library against the oracle's
processing variant (reading R15 in ``oracle/spec_verify_oracle.c``).

Sequences whose nucleus cut is a near tie in fp64 (the running sum within
1e-5 of top_p at a step, see ``paritylib.nucleus_near_cut``), or whose
decisions lie within 1e-5 of a threshold, are counted and left out; the rest
must match exactly, with p and q within 1e-5 at every position.
"""
import numpy as np
import pytest

import oracle
import workloads
from paritylib import DECISION_TOL, PROB_TOL, nucleus_near_cut, to_dev

pytestmark = pytest.mark.gpu


def _inputs(name, seed, B, top_p_range=(0.6, 0.95), **over):
    case = workloads.make_case(name, seed=seed, B=B, **over)
    pr = workloads.make_processors(seed, B, case.V, top_p=top_p_range)
    temp_rows = np.repeat(case.temperature, case.k).reshape(B, case.k)
    drafts = oracle.sample_rows_procs(case.draft, case.draft_uniforms, temp_rows, case.top_k, top_p=pr.top_p)
    return case, pr.top_p, drafts.astype(np.int32)


def _run_gpu(case, drafts, top_p, **opt):
    import torch

    import draft_token_verification_verify_b200 as sv

    dev = torch.device("cuda:0")
    B, k = case.B, case.k
    tp = None if top_p is None else torch.from_numpy(np.ascontiguousarray(top_p, np.float32)).to(dev)
    out_p = torch.full((B, k), float("nan"), dtype=torch.float32, device=dev)
    out_q = torch.full((B, k), float("nan"), dtype=torch.float32, device=dev)
    tok, n = sv.verify(to_dev(case.target), to_dev(case.draft), torch.from_numpy(drafts).to(dev),
                       to_dev(case.uniforms), to_dev(case.temperature), case.top_k, out_p=out_p, out_q=out_q,
                       opts=sv.make_options(top_p=tp, **opt))
    torch.cuda.synchronize()
    return tok.cpu().numpy(), n.cpu().numpy(), out_p.cpu().numpy(), out_q.cpu().numpy()


def _near_cut(case, b, top_p):
    T = float(case.temperature[b])
    rows = [case.target[b, i] for i in range(case.k + 1)] + [case.draft[b, i] for i in range(case.k)]
    return any(nucleus_near_cut(oracle.process_row(r, T, case.top_k), float(top_p[b])) for r in rows)


def _check(case, top_p, drafts, gpu):
    tok, n, p, q = gpu
    ref = oracle.verify_procs(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k,
                              top_p=top_p)
    k, skipped = case.k, 0
    for b in range(case.B):
        u = case.uniforms[b]
        j = ref.n_accepted[b]
        near = _near_cut(case, b, top_p)
        near |= any(abs(float(u[i]) - ref.ratio[b, i]) < DECISION_TOL for i in range(min(j + 1, k)))
        near |= j >= 0 and (abs(float(u[k]) - ref.cdf_lo[b]) < DECISION_TOL or abs(float(u[k]) - ref.cdf_hi[b]) < DECISION_TOL)
        if near:
            skipped += 1
            continue
        assert n[b] == j, (b, n[b], j)
        assert np.array_equal(tok[b], ref.tokens[b]), (b, tok[b], ref.tokens[b])
        if j >= 0:
            assert np.max(np.abs(p[b] - ref.p[b])) <= PROB_TOL, (b, p[b], ref.p[b])
            assert np.max(np.abs(q[b] - ref.q[b])) <= PROB_TOL, (b, q[b], ref.q[b])
    assert skipped <= max(1, case.B // 4), skipped
    return ref


def test_top_p_batched_full_vocabulary():
    case, top_p, drafts = _inputs("batched", 51, 16)
    ref = _check(case, top_p, drafts, _run_gpu(case, drafts, top_p))
    assert ref.errors == 0


@pytest.mark.parametrize("chunks", [1, 3])
def test_top_p_chunked_rows(chunks):
    case, top_p, drafts = _inputs("batched", 52 + chunks, 6, V=30011)
    _check(case, top_p, drafts, _run_gpu(case, drafts, top_p, chunks_per_row=chunks))


def test_top_p_fp32():
    case, top_p, drafts = _inputs("large", 55, 6, top_k=40, V=20000)
    _check(case, top_p, drafts, _run_gpu(case, drafts, top_p))


def test_top_p_one_is_no_nucleus():
    case, _, drafts = _inputs("batched", 56, 8, V=30011)
    ones = np.ones(case.B, np.float32)
    a = _run_gpu(case, drafts, ones)
    b = _run_gpu(case, drafts, None)
    for x, y in zip(a, b):
        assert np.array_equal(x, y, equal_nan=True)


def test_top_p_out_of_range_is_a_row_error():
    case, top_p, drafts = _inputs("batched", 57, 4, V=3001)
    top_p = np.array([0.0, 1.5, 0.9, np.nan], np.float32)
    tok, n, _, _ = _run_gpu(case, drafts, top_p)
    assert n[0] == -1 and n[1] == -1 and n[3] == -1 and n[2] >= 0
    assert np.all(tok[[0, 1, 3]] == -1)


def test_greedy_takes_no_nucleus():
    import torch

    import draft_token_verification_verify_b200 as sv

    case = workloads.make_case("greedy", seed=58, B=2, V=500)
    dev = torch.device("cuda:0")
    tp = torch.full((2,), 0.9, dtype=torch.float32, device=dev)
    tok = torch.empty((2, case.k + 1), dtype=torch.int32, device=dev)
    n = torch.empty((2,), dtype=torch.int32, device=dev)
    st = sv.spec_verify_ex(to_dev(case.target), None, torch.zeros((2, case.k), dtype=torch.int32, device=dev),
                           None, 2, case.k, case.V, None, 0, sv.SV_MODE_GREEDY | sv.SV_DTYPE_BF16, tok, n,
                           opts=sv.make_options(top_p=tp))
    assert st == sv.SV_ERR_UNSUPPORTED
