"""Vocabulary mask and repetition penalty on the GPU against the oracle's
processing variant (readings R12-R14 in ``oracle/spec_verify_oracle.c``):
section "提议与核验的基本步骤", paragraph 4, of the speculative decoding entry
"推测解码" requires every processing rule in effect to act on the target and
the draft distributions alike.

Each case draws its drafts from the processed draft distribution (the
oracle's sampler), verifies on the GPU and compares with
``oracle.verify_procs`` under the usual rule: tokens and counts bit-exact
except near-threshold decisions (counted and window-checked), p and q within
1e-5 at every position, error rows identical.  The GPU proposer draw with the
same processors is compared with ``oracle.sample_rows_procs``.
"""
import numpy as np
import pytest

import draft_token_verification_verify_b200 as sv
import oracle
import workloads
from paritylib import compare, compare_samples, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    import __graft_entry__

    __graft_entry__.build()
    return cuda_device


def _procs(seed, B, V, which, theta=1.3, n_rep=48, allowed=0.5):
    pr = workloads.make_processors(seed, B, V, top_p=1.0, rep_penalty=theta, n_rep=n_rep,
                                   allowed_fraction=allowed)
    d = {"top_p": None, "rep_penalty": None, "rep_ids": None, "mask": None}
    if "mask" in which:
        d["mask"] = pr.mask
    if "penalty" in which:
        d["rep_penalty"] = pr.rep_penalty
        d["rep_ids"] = pr.rep_ids
    return d


def _dev_procs(d):
    import torch

    dev = torch.device("cuda:0")
    t = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    return dict(vocab_mask=t(d["mask"], np.int32), rep_ids=t(d["rep_ids"], np.int32),
                rep_penalty=t(d["rep_penalty"], np.float32))


def _oracle_drafts(case, d):
    temp_rows = np.repeat(case.temperature, case.k).reshape(case.B, case.k)
    return oracle.sample_rows_procs(case.draft, case.draft_uniforms, temp_rows, case.top_k,
                                    rep_penalty=d["rep_penalty"], rep_ids=d["rep_ids"],
                                    mask=d["mask"]).astype(np.int32)


def _verify_gpu(case, drafts, d, **opt):
    import torch

    dev = torch.device("cuda:0")
    B, k = case.B, case.k
    out_p = torch.full((B, k), float("nan"), dtype=torch.float32, device=dev)
    out_q = torch.full((B, k), float("nan"), dtype=torch.float32, device=dev)
    status = torch.full((1,), 12345, dtype=torch.int32, device=dev)
    keep = _dev_procs(d)
    tok, n = sv.verify(to_dev(case.target), to_dev(case.draft), torch.from_numpy(drafts).to(dev),
                       to_dev(case.uniforms), to_dev(case.temperature), case.top_k, out_p=out_p, out_q=out_q,
                       out_status=status, opts=sv.make_options(**keep, **opt))
    torch.cuda.synchronize()
    from paritylib import GpuResult

    return GpuResult(tok.cpu().numpy(), n.cpu().numpy(), out_p.cpu().numpy(), out_q.cpu().numpy(),
                     int(status.cpu().item()))


def _check(case, d, drafts=None, **opt):
    if drafts is None:
        drafts = _oracle_drafts(case, d)
    ref = oracle.verify_procs(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k,
                              rep_penalty=d["rep_penalty"], rep_ids=d["rep_ids"], mask=d["mask"])
    gpu = _verify_gpu(case, drafts, d, **opt)
    assert gpu.status == 0, gpu.status
    rep = compare(ref, gpu, case.uniforms,
                  inputs=(case.target, case.draft, drafts, case.temperature, case.top_k, d))
    print(rep)
    assert rep.flagged_accept <= max(1, 0.01 * rep.sequences), rep
    return ref, gpu, rep


@pytest.mark.parametrize("which", ["mask", "penalty", "mask+penalty"])
def test_batched_top_k_full_vocabulary(which):
    """bf16, V = 151,936, T = 0.7, top-k 50 (the batched workload's value model)."""
    case = workloads.make_case("batched", seed=61, B=12)
    ref, _, rep = _check(case, _procs(61, case.B, case.V, which))
    assert ref.errors == 0 and rep.exact >= case.B - 2


def test_penalty_below_one_with_top_k():
    """theta < 1 raises the listed positive logits: the streaming pass cannot
    skip a vector on its raw maximum then."""
    case = workloads.make_case("batched", seed=72, B=8)
    ref, _, rep = _check(case, _procs(72, case.B, case.V, "mask+penalty", theta=0.6, n_rep=400))
    assert ref.errors == 0 and rep.exact >= case.B - 2


@pytest.mark.parametrize("which", ["mask", "mask+penalty"])
def test_softmax_full_vocabulary_bf16(which):
    """No top-k: the residual draws rescan the processed row pair."""
    case = workloads.make_case("single", seed=62, B=6)
    _check(case, _procs(62, case.B, case.V, which, theta=0.8))


@pytest.mark.parametrize("top_k", [0, 40])
def test_fp32_mixed_temperatures(top_k):
    """fp32, V = 128,256, T in {0.5, 1.0, 1.5} (the large workload's value model)."""
    case = workloads.make_case("large", seed=63, B=8, top_k=top_k)
    _check(case, _procs(63, case.B, case.V, "mask+penalty", theta=1.7))


@pytest.mark.parametrize("chunks", [1, 3])
def test_ragged_vocabulary_and_chunked_rows(chunks):
    """V = 30,011: rows not 16-byte aligned, mask words straddling vectors."""
    case = workloads.make_case("batched", seed=64 + chunks, B=5, V=30011)
    _check(case, _procs(64, case.B, case.V, "mask+penalty", allowed=0.3), chunks_per_row=chunks)


def test_radix_top_k_path():
    case = workloads.make_case("batched", seed=66, B=4, V=30011)
    _check(case, _procs(66, case.B, case.V, "mask+penalty"), topk_path=2)


def test_heavy_penalty_list():
    """Many listed ids (with repeats and ids outside [0, V)), strong penalty."""
    case = workloads.make_case("batched", seed=67, B=4, V=20000)
    d = _procs(67, case.B, case.V, "penalty", theta=3.0, n_rep=2000)
    ids = d["rep_ids"].copy()
    ids[:, ::7] = ids[:, 1::7][:, : ids[:, ::7].shape[1]]  # repeats
    ids[:, 3] = -5
    ids[:, 5] = case.V + 3
    d["rep_ids"] = ids
    _check(case, d)


def test_unit_penalty_is_no_penalty():
    case = workloads.make_case("batched", seed=68, B=4, V=30011)
    drafts = oracle.draft_tokens_for(case)
    d = _procs(68, case.B, case.V, "penalty", theta=1.0)
    a = _verify_gpu(case, drafts, d)
    b = _verify_gpu(case, drafts, {"top_p": None, "rep_penalty": None, "rep_ids": None, "mask": None})
    assert np.array_equal(a.tokens, b.tokens) and np.array_equal(a.n_accepted, b.n_accepted)
    assert np.array_equal(a.p, b.p) and np.array_equal(a.q, b.q)


@pytest.mark.parametrize("what", ["all_masked", "theta_zero", "theta_negative", "theta_nan", "theta_inf",
                                  "nan_logit_masked"])
def test_row_errors(what):
    case = workloads.make_case("batched", seed=69, B=3, V=4099)
    d = _procs(69, case.B, case.V, "mask+penalty")
    drafts = _oracle_drafts(case, d)
    target = case.target.copy()
    if what == "all_masked":
        d["mask"][0, :] = 0
    elif what.startswith("theta"):
        d["rep_penalty"][0] = {"theta_zero": 0.0, "theta_negative": -1.0, "theta_nan": np.nan,
                               "theta_inf": np.inf}[what]
    elif what == "nan_logit_masked":
        v = int(np.flatnonzero(~oracle.process_row_procs(target[0, 1], mask=d["mask"][0]).astype(bool))[0])
        target[0, 1, v] = 0x7fc0  # bf16 NaN at a disallowed token: still a row error
    case.target = target
    ref, gpu, _ = _check(case, d, drafts=drafts)
    assert ref.n_accepted[0] == -1 and gpu.n_accepted[0] == -1
    assert ref.n_accepted[1] >= 0 and ref.n_accepted[2] >= 0


def test_greedy_takes_no_processors():
    import torch

    case = workloads.make_case("greedy", seed=70, B=2, V=500)
    dev = torch.device("cuda:0")
    keep = _dev_procs(_procs(70, case.B, case.V, "mask"))
    tok = torch.empty((2, case.k + 1), dtype=torch.int32, device=dev)
    n = torch.empty((2,), dtype=torch.int32, device=dev)
    st = sv.spec_verify_ex(to_dev(case.target), None, torch.zeros((2, case.k), dtype=torch.int32, device=dev),
                           None, 2, case.k, case.V, None, 0, sv.SV_MODE_GREEDY | sv.SV_DTYPE_BF16, tok, n,
                           opts=sv.make_options(**keep))
    assert st == sv.SV_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,top_k", [("batched", 50), ("batched", 0), ("large", 0)])
def test_sampler_with_processors(name, top_k):
    """The proposer's draw: k rows per sequence share the sequence's processors."""
    import torch

    case = workloads.make_case(name, seed=71, B=6, top_k=top_k, V=None if name == "batched" else 40000)
    d = _procs(71, case.B, case.V, "mask+penalty")
    k = case.k
    temp_rows = np.repeat(case.temperature, k)
    logits = case.draft.reshape(case.B * k, case.V)
    u = case.draft_uniforms.reshape(-1)
    keep = _dev_procs(d)
    got = sv.sample(to_dev(logits), to_dev(u), to_dev(temp_rows), top_k,
                    opts=sv.make_options(rows_per_sequence=k, **keep))
    torch.cuda.synchronize()
    ref = oracle.sample_rows_procs(case.draft, case.draft_uniforms, temp_rows.reshape(case.B, k), top_k,
                                   rep_penalty=d["rep_penalty"], rep_ids=d["rep_ids"], mask=d["mask"]).reshape(-1)
    # the CDF points of the oracle's draws, for the near-threshold rule
    lo = np.empty(ref.size)
    hi = np.empty(ref.size)
    from paritylib import process, seq_procs

    for r in range(ref.size):
        w = process(logits[r], float(temp_rows[r]), top_k, seq_procs(d, r // k))
        C = np.cumsum(w) / w.sum()
        y = int(ref[r])
        lo[r] = C[y - 1] if y > 0 else 0.0
        hi[r] = C[y]
    rep = compare_samples(logits, u, temp_rows, top_k, got.cpu().numpy(), ref, lo, hi, procs=d, rows_per_seq=k)
    print(rep)
    assert rep.exact + rep.flagged == ref.size
